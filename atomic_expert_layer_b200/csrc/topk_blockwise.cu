// topk_blockwise.cu -- the pages' own form of the global top-K: the implicit
// N_r x N_c score grid is cut into blocks, each block goes to a GPU thread
// block that keeps its local top-K, and the local results are merged.
//
// "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale"
// (rainbus review page, method paragraph, step 2): S_ij = p_r[i] + p_c[j]
// is never materialised; a parallel top-K assigns blocks of the implicit grid
// to thread blocks and extracts the global top-K expert indices.
//
// This is the alternative to the row / column top-K + candidate merge of
// topk.cu, which prunes the grid to the (a+1)(b+1) <= K cells first.  Here
// every cell is scored: the cost is L * N_r * N_c fp32 adds instead of
// L * (N_r + N_c) selections plus ~K ln K candidates.  Results are identical
// (same fp32 S, same order key (S desc, p_r desc, p_c desc, n asc), same
// gate formula).
//
// Kernel 1 (band): CTA (token t, band b) streams grid rows
//   [b * rows, (b + 1) * rows) x all columns.  A cell enters a shared-memory
//   buffer only if key(S) >= T, the key of the current K-th best (equal keys
//   are kept: the secondary keys may still rank them in).  When the buffer
//   could overflow it is bitonic-sorted by the full key and cut to K, which
//   raises T.  The band's top-K (sentinel-padded) goes to global memory.
// Kernel 2 (merge): CTA per token sorts the bands' candidates, keeps K and
//   computes the gates (softmax over the K selected S).
#include "omni_common.cuh"
#include "omni_internal.h"

namespace omni {
namespace {

constexpr int kBandThreads = 256;
constexpr int kBandBuf = 2048;           // candidate buffer (entries), power of two
constexpr int kColChunk = 1024;          // columns scanned between overflow checks

struct Cell {            // one grid cell; larger key ranks first
    uint32_t skey;       // key(S)
    uint32_t prkey;      // key(p_r[i])
    uint32_t pckey;      // key(p_c[j])
    uint32_t n;          // i * N_c + j
};

__device__ __forceinline__ bool cell_before(const Cell &u, const Cell &v) {
    if (u.skey != v.skey) return u.skey > v.skey;
    if (u.prkey != v.prkey) return u.prkey > v.prkey;
    if (u.pckey != v.pckey) return u.pckey > v.pckey;
    return u.n < v.n;
}

__device__ __forceinline__ Cell sentinel() {   // after every real cell
    Cell c;
    c.skey = 0u; c.prkey = 0u; c.pckey = 0u; c.n = 0xffffffffu;
    return c;
}

// Sorts buf[0, n2) (n2 a power of two) best-first; all threads of the CTA.
__device__ void bitonic_sort_cells(Cell *buf, int n2) {
    for (int k = 2; k <= n2; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < n2; i += blockDim.x) {
                const int l = i ^ j;
                if (l > i) {
                    const Cell a = buf[i], b = buf[l];
                    // ascending blocks hold best-first order
                    const bool best_first = (i & k) == 0;
                    const bool swap = best_first ? cell_before(b, a) : cell_before(a, b);
                    if (swap) {
                        buf[i] = b;
                        buf[l] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
}

__host__ __device__ __forceinline__ int pow2_at_least(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

// Sort the cnt buffered cells, keep the best min(cnt, K); returns the new
// count and sets *T to the K-th best key(S) once K cells are held.
__device__ int compact_cells(Cell *buf, int cnt, int K, uint32_t *T) {
    const int n2 = pow2_at_least(cnt > 1 ? cnt : 2);
    for (int i = cnt + (int)threadIdx.x; i < n2; i += blockDim.x) buf[i] = sentinel();
    __syncthreads();
    bitonic_sort_cells(buf, n2);
    const int keep = cnt < K ? cnt : K;
    if (keep == K) *T = buf[K - 1].skey;
    return keep;
}

__global__ void __launch_bounds__(kBandThreads)
grid_band_topk_kernel(const float *__restrict__ p_r, const float *__restrict__ p_c, int L,
                      int N_r, int N_c, int K, int rows, int nb, Cell *__restrict__ out) {
    extern __shared__ __align__(16) uint8_t smem[];
    Cell *buf = reinterpret_cast<Cell *>(smem);
    float *pc_s = reinterpret_cast<float *>(buf + kBandBuf);       // N_c
    float *pr_s = pc_s + N_c;                                        // rows
    __shared__ int cnt;
    __shared__ uint32_t T;
    grid_dependency_wait();
    grid_dependents_launch();
    const int t = blockIdx.x / nb;
    const int b = blockIdx.x % nb;
    if (t >= L) return;                                  // the same in every thread
    const int r0 = b * rows;
    const int r1 = r0 + rows < N_r ? r0 + rows : N_r;
    for (int j = threadIdx.x; j < N_c; j += blockDim.x) pc_s[j] = p_c[(size_t)t * N_c + j];
    for (int i = threadIdx.x; i < r1 - r0; i += blockDim.x) pr_s[i] = p_r[(size_t)t * N_r + r0 + i];
    if (threadIdx.x == 0) {
        cnt = 0;
        T = 0u;                                          // every key is >= 0
    }
    __syncthreads();
    for (int i = r0; i < r1; ++i) {
        const float pr = pr_s[i - r0];
        const uint32_t prk = f2key(pr);
        for (int j0 = 0; j0 < N_c; j0 += kColChunk) {
            // every thread reads the count before any thread appends to it,
            // so all take the same branch (and meet the same barriers)
            const int c = cnt;
            __syncthreads();
            if (c + kColChunk > kBandBuf) {
                uint32_t tn = T;
                const int kept = compact_cells(buf, c, K, &tn);
                __syncthreads();
                if (threadIdx.x == 0) {
                    cnt = kept;
                    T = tn;
                }
                __syncthreads();
            }
            const uint32_t thr = T;
            const int j1 = j0 + kColChunk < N_c ? j0 + kColChunk : N_c;
            for (int j = j0 + (int)threadIdx.x; j < j1; j += blockDim.x) {
                const float S = __fadd_rn(pr, pc_s[j]);
                const uint32_t sk = f2key(S);
                if (sk >= thr) {
                    const int pos = atomicAdd(&cnt, 1);
                    Cell cell;
                    cell.skey = sk;
                    cell.prkey = prk;
                    cell.pckey = f2key(pc_s[j]);
                    cell.n = (uint32_t)i * (uint32_t)N_c + (uint32_t)j;
                    buf[pos] = cell;
                }
            }
            __syncthreads();
        }
    }
    const int c = cnt;
    __syncthreads();
    uint32_t tn = T;
    const int kept = compact_cells(buf, c, K, &tn);
    Cell *o = out + ((size_t)t * nb + b) * K;
    for (int k = threadIdx.x; k < K; k += blockDim.x) o[k] = k < kept ? buf[k] : sentinel();
}

__global__ void __launch_bounds__(kBandThreads)
grid_band_merge_kernel(const Cell *__restrict__ cand, int L, int K, int nb,
                       int32_t *__restrict__ idx, float *__restrict__ score,
                       float *__restrict__ gate) {
    extern __shared__ __align__(16) uint8_t smem[];
    Cell *buf = reinterpret_cast<Cell *>(smem);
    grid_dependency_wait();
    grid_dependents_launch();
    const int t = blockIdx.x;
    if (t >= L) return;
    const int n = nb * K;
    const int n2 = pow2_at_least(n > 1 ? n : 2);
    for (int i = threadIdx.x; i < n2; i += blockDim.x)
        buf[i] = i < n ? cand[(size_t)t * n + i] : sentinel();
    __syncthreads();
    bitonic_sort_cells(buf, n2);
    if (threadIdx.x < 32) {
        // gates: softmax over the K selected S (buf[0] holds the maximum)
        const unsigned lane = lane_id();
        const float smx = key2f(buf[0].skey);
        float part = 0.f;
        for (int k = lane; k < K; k += 32) part += expf(key2f(buf[k].skey) - smx);
        const float den = warp_sum(part);
        for (int k = lane; k < K; k += 32) {
            const float S = key2f(buf[k].skey);
            idx[(size_t)t * K + k] = (int32_t)buf[k].n;
            score[(size_t)t * K + k] = S;
            gate[(size_t)t * K + k] = expf(S - smx) / den;
        }
    }
}

}  // namespace

// Bands per token (0: the candidates do not fit, the call is unsupported).
int blockwise_bands(int N_r, int N_c, int K) {
    // the bands' candidates (16 bytes each) live in the 4 (N_r + N_c) bytes
    // per token of the logits area, which log-probability input leaves unused
    int nb = (N_r + N_c) / (4 * K);
    if (nb > N_r) nb = N_r;
    if (nb > 64) nb = 64;
    return nb;
}

cudaError_t launch_topk_blockwise(const float *p_r, const float *p_c, int L, int N_r, int N_c,
                                  int K, void *cand, int32_t *idx, float *score, float *gate,
                                  cudaStream_t st) {
    const int nb = blockwise_bands(N_r, N_c, K);
    const int rows = (N_r + nb - 1) / nb;
    const size_t band_smem = sizeof(Cell) * kBandBuf + 4 * (size_t)N_c + 4 * (size_t)rows;
    const size_t merge_smem = sizeof(Cell) * (size_t)pow2_at_least(nb * K > 1 ? nb * K : 2);
    cudaError_t e = cudaFuncSetAttribute(grid_band_topk_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)band_smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(grid_band_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)merge_smem);
    if (e != cudaSuccess) return e;
    Cell *c = static_cast<Cell *>(cand);
    e = launch(grid_band_topk_kernel, dim3((unsigned)((int64_t)L * nb)), dim3(kBandThreads),
               band_smem, st, p_r, p_c, L, N_r, N_c, K, rows, nb, c);
    if (e != cudaSuccess) return e;
    return launch(grid_band_merge_kernel, dim3((unsigned)L), dim3(kBandThreads), merge_smem, st,
                  (const Cell *)c, L, K, nb, idx, score, gate);
}

}  // namespace omni

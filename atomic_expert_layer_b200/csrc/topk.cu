// topk.cu -- Cartesian product router selection on sm_100a.
//
// "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale"
// (rainbus review page, method paragraph, step 2): p_r, p_c are the
// LogSoftmax of the row and column logits and the score of expert (i, j) is
// S_ij = p_r[i] + p_c[j]; the global top-K is taken without building the
// N_r x N_c grid.  The order key is (S desc, p_r desc, p_c desc, n asc) with
// n = i * N_c + j, and axis ranks use (p desc, index asc).  Gates are the
// softmax over the K selected scores.
//
// Kernel 1 (axis_topk): one warp per (token, axis).  Optional LogSoftmax,
//   then an exact radix select (4 passes of 8 bits over order-preserving
//   keys) of the axis' top min(K, n) entries, then a rank sort of those.
// Kernel 2 (merge_topk): one warp per token.  Because fp32 addition is
//   monotone, a cell with row rank a and column rank b is dominated by every
//   cell (a', b') with a' <= a, b' <= b, and the key above ranks a dominating
//   cell first even on equal S; so the K best cells all satisfy
//   (a+1)(b+1) <= K.  Those C candidates (C = sum_a min(Kc, K/(a+1))) are
//   scored, radix-selected on S and rank-sorted by the full key.
#include "omni_common.cuh"
#include "omni_internal.h"

namespace omni {
namespace {

// Exact k-th largest key of keys[0..n) (a warp, smem histogram `hist` of 256).
// Returns the threshold key T and sets *take_eq to how many keys equal to T
// belong to the top k (the rest of the top k is every key > T).
__device__ uint32_t warp_radix_select(const uint32_t *keys, int n, int k, uint32_t *hist,
                                      int *take_eq) {
    const unsigned lane = lane_id();
    uint32_t prefix = 0, mask = 0;
    int krem = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = lane; b < 256; b += 32) hist[b] = 0;
        __syncwarp();
        for (int i = lane; i < n; i += 32) {
            const uint32_t key = keys[i];
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncwarp();
        // lane l owns bins 255-8l down to 248-8l
        int c[8], tot = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            c[j] = (int)hist[255 - 8 * lane - j];
            tot += c[j];
        }
        const int incl = warp_iscan(tot);
        const int excl = incl - tot;
        const bool mine = excl < krem && krem <= incl;
        const unsigned bal = __ballot_sync(0xffffffffu, mine);
        int digit = 0, above = 0;
        if (mine) {
            int run = excl;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (run + c[j] >= krem) {
                    digit = 255 - 8 * (int)lane - j;
                    above = run;
                    break;
                }
                run += c[j];
            }
        }
        const int src = __ffs(bal) - 1;
        digit = __shfl_sync(0xffffffffu, digit, src);
        above = __shfl_sync(0xffffffffu, above, src);
        krem -= above;
        prefix |= (uint32_t)digit << shift;
        mask |= 255u << shift;
        __syncwarp();
    }
    *take_eq = krem;
    return prefix;
}

// ------------------------------------------------------------ axis top-K
// Dynamic smem per warp: keys[nmax] + hist[256] + sel_key[kmax] + sel_idx[kmax].
__global__ void axis_topk_kernel(const float *__restrict__ in_r, const float *__restrict__ in_c,
                                 int logsoftmax, float *__restrict__ p_r_out,
                                 float *__restrict__ p_c_out, int L, int N_r, int N_c, int K,
                                 float *__restrict__ row_val, int *__restrict__ row_idx,
                                 float *__restrict__ col_val, int *__restrict__ col_idx,
                                 int nmax, int kmax) {
    extern __shared__ __align__(16) uint32_t smem_u[];
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    const int wpb = blockDim.x >> 5;
    const int64_t prob = (int64_t)blockIdx.x * wpb + warp;
    if (prob >= 2 * (int64_t)L) return;
    const int t = (int)(prob >> 1);
    const int axis = (int)(prob & 1);
    const int n = axis ? N_c : N_r;
    const int kx = K < n ? K : n;
    const float *in = (axis ? in_c : in_r) + (size_t)t * n;
    float *pout = axis ? p_c_out : p_r_out;
    float *oval = (axis ? col_val : row_val) + (size_t)t * kx;
    int *oidx = (axis ? col_idx : row_idx) + (size_t)t * kx;

    uint32_t *keys = smem_u + (size_t)warp * (nmax + 256 + 2 * kmax);
    uint32_t *hist = keys + nmax;
    uint32_t *sel_key = hist + 256;
    int *sel_idx = reinterpret_cast<int *>(sel_key + kmax);

    if (logsoftmax) {
        float mx = -INFINITY;
        for (int i = lane; i < n; i += 32) {
            const float v = in[i];
            keys[i] = __float_as_uint(v);
            mx = fmaxf(mx, v);
        }
        mx = warp_max(mx);
        float sum = 0.f;
        for (int i = lane; i < n; i += 32) sum += expf(__uint_as_float(keys[i]) - mx);
        sum = warp_sum(sum);
        const float lse = mx + logf(sum);
        for (int i = lane; i < n; i += 32) {
            const float p = __uint_as_float(keys[i]) - lse;
            if (pout) pout[(size_t)t * n + i] = p;
            keys[i] = f2key(p);
        }
    } else {
        for (int i = lane; i < n; i += 32) keys[i] = f2key(in[i]);
    }
    __syncwarp();

    int take_eq;
    const uint32_t T = warp_radix_select(keys, n, kx, hist, &take_eq);

    // collect the top kx in index order: every key > T, and the first take_eq keys == T
    int taken = 0, eq_seen = 0;
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + (int)lane;
        const uint32_t key = i < n ? keys[i] : 0u;
        const bool gt = i < n && key > T;
        const bool eq = i < n && key == T;
        const unsigned beq = __ballot_sync(0xffffffffu, eq);
        const int eq_rank = eq_seen + __popc(beq & lanemask_lt());
        const bool take = gt || (eq && eq_rank < take_eq);
        const unsigned bt = __ballot_sync(0xffffffffu, take);
        if (take) {
            const int pos = taken + __popc(bt & lanemask_lt());
            sel_key[pos] = key;
            sel_idx[pos] = i;
        }
        taken += __popc(bt);
        eq_seen += __popc(beq);
    }
    __syncwarp();
    // rank sort by (key desc, index asc); sel is in index order
    for (int u = lane; u < kx; u += 32) {
        const uint32_t ku = sel_key[u];
        int r = 0;
        for (int v = 0; v < kx; ++v) {
            const uint32_t kv = sel_key[v];
            r += (kv > ku) | ((kv == ku) & (v < u));
        }
        oval[r] = key2f(ku);
        oidx[r] = sel_idx[u];
    }
}

// ----------------------------------------------------------- merge top-K
struct Cand {          // one grid cell of the candidate block
    uint32_t skey;     // key(S)
    uint32_t prkey;    // key(p_r[i])
    uint32_t pckey;    // key(p_c[j])
    uint32_t n;        // i * N_c + j
};

// true if cell u ranks before cell v
__device__ __forceinline__ bool better(const Cand &u, const Cand &v) {
    if (u.skey != v.skey) return u.skey > v.skey;
    if (u.prkey != v.prkey) return u.prkey > v.prkey;
    if (u.pckey != v.pckey) return u.pckey > v.pckey;
    return u.n < v.n;
}

// Dynamic smem per warp:
//   rv[Kr] f32, ri[Kr] i32, cv[Kc] f32, ci[Kc] i32, ckey[C] u32, cab[C] u32,
//   hist[256] u32, q[C] Cand, out_S[K] f32, out_n[K] u32
__global__ void merge_topk_kernel(const float *__restrict__ row_val,
                                  const int *__restrict__ row_idx,
                                  const float *__restrict__ col_val,
                                  const int *__restrict__ col_idx, int L, int N_c, int K, int Kr,
                                  int Kc, int C, size_t warp_words, int32_t *__restrict__ idx,
                                  float *__restrict__ score, float *__restrict__ gate) {
    extern __shared__ __align__(16) uint32_t smem_u[];
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    const int t = blockIdx.x * (blockDim.x >> 5) + warp;
    if (t >= L) return;
    uint32_t *base = smem_u + (size_t)warp * warp_words;
    float *rv = reinterpret_cast<float *>(base);
    uint32_t *ri = base + Kr;
    float *cv = reinterpret_cast<float *>(ri + Kr);
    uint32_t *ci = reinterpret_cast<uint32_t *>(cv + Kc);
    uint32_t *ckey = ci + Kc;
    uint32_t *cab = ckey + C;
    uint32_t *hist = cab + C;
    const size_t q_off = ((size_t)(2 * Kr + 2 * Kc + 2 * C + 256) + 3) & ~(size_t)3;
    Cand *q = reinterpret_cast<Cand *>(base + q_off);
    float *out_S = reinterpret_cast<float *>(q + C);
    uint32_t *out_n = reinterpret_cast<uint32_t *>(out_S + K);

    for (int a = lane; a < Kr; a += 32) {
        rv[a] = row_val[(size_t)t * Kr + a];
        ri[a] = (uint32_t)row_idx[(size_t)t * Kr + a];
    }
    for (int b = lane; b < Kc; b += 32) {
        cv[b] = col_val[(size_t)t * Kc + b];
        ci[b] = (uint32_t)col_idx[(size_t)t * Kc + b];
    }
    __syncwarp();
    // candidate block: a-major, b < min(Kc, K / (a+1))
    int off = 0;
    for (int a = 0; a < Kr; ++a) {
        int nb = K / (a + 1);
        if (nb > Kc) nb = Kc;
        if (nb <= 0) break;
        const float pr = rv[a];
        for (int b = lane; b < nb; b += 32) {
            const float S = __fadd_rn(pr, cv[b]);
            ckey[off + b] = f2key(S);
            cab[off + b] = ((uint32_t)a << 16) | (uint32_t)b;
        }
        off += nb;
    }
    __syncwarp();

    int take_eq;
    const uint32_t T = warp_radix_select(ckey, C, K, hist, &take_eq);

    // Q = all candidates with key(S) >= T, in candidate order
    int nq = 0;
    for (int c0 = 0; c0 < C; c0 += 32) {
        const int c = c0 + (int)lane;
        const bool in = c < C && ckey[c] >= T;
        const unsigned bal = __ballot_sync(0xffffffffu, in);
        if (in) {
            const int pos = nq + __popc(bal & lanemask_lt());
            const uint32_t ab = cab[c];
            const int a = (int)(ab >> 16), b = (int)(ab & 0xffffu);
            Cand cd;
            cd.skey = ckey[c];
            cd.prkey = f2key(rv[a]);
            cd.pckey = f2key(cv[b]);
            cd.n = ri[a] * (uint32_t)N_c + ci[b];
            q[pos] = cd;
        }
        nq += __popc(bal);
    }
    __syncwarp();
    // rank by the full key; the K best go to out[rank]
    for (int u = lane; u < nq; u += 32) {
        const Cand cu = q[u];
        int r = 0;
        for (int v = 0; v < nq; ++v) r += better(q[v], cu) ? 1 : 0;
        if (r < K) {
            out_S[r] = key2f(cu.skey);
            out_n[r] = cu.n;
        }
    }
    __syncwarp();
    // gates: softmax over the K selected S (S sorted, out_S[0] is the max)
    const float smax = out_S[0];
    float part = 0.f;
    for (int k = lane; k < K; k += 32) part += expf(out_S[k] - smax);
    const float den = warp_sum(part);
    for (int k = lane; k < K; k += 32) {
        const float S = out_S[k];
        idx[(size_t)t * K + k] = (int32_t)out_n[k];
        score[(size_t)t * K + k] = S;
        gate[(size_t)t * K + k] = expf(S - smax) / den;
    }
}

}  // namespace

int merge_candidates(int K, int Kr, int Kc) {
    int C = 0;
    for (int a = 0; a < Kr; ++a) {
        int nb = K / (a + 1);
        if (nb > Kc) nb = Kc;
        if (nb <= 0) break;
        C += nb;
    }
    return C;
}

cudaError_t launch_axis_topk(const float *in_r, const float *in_c, bool logsoftmax,
                             float *p_r_out, float *p_c_out, int L, int N_r, int N_c, int K,
                             float *row_val, int *row_idx, float *col_val, int *col_idx,
                             int *status, cudaStream_t st) {
    (void)status;
    const int nmax = N_r > N_c ? N_r : N_c;
    const int kmax = K < nmax ? K : nmax;
    const size_t per_warp = (size_t)(nmax + 256 + 2 * kmax) * 4;
    int wpb = (int)((96 * 1024) / per_warp);
    if (wpb > 8) wpb = 8;
    if (wpb < 1) wpb = 1;
    const size_t smem = per_warp * wpb;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(axis_topk_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t probs = 2 * (int64_t)L;
    const unsigned grid = (unsigned)((probs + wpb - 1) / wpb);
    axis_topk_kernel<<<grid, 32 * wpb, smem, st>>>(in_r, in_c, logsoftmax ? 1 : 0, p_r_out,
                                                   p_c_out, L, N_r, N_c, K, row_val, row_idx,
                                                   col_val, col_idx, nmax, kmax);
    return cudaGetLastError();
}

cudaError_t launch_merge_topk(const float *row_val, const int *row_idx, const float *col_val,
                              const int *col_idx, int L, int N_c, int K, int Kr, int Kc, int C,
                              int32_t *idx, float *score, float *gate, cudaStream_t st) {
    // words per warp: rv, ri (Kr each), cv, ci (Kc each), ckey, cab (C each),
    // hist 256, q (4 words per cand), out_S, out_n (K each); pad to 4 words
    size_t words = 2 * (size_t)Kr + 2 * (size_t)Kc + 2 * (size_t)C + 256;
    words = (words + 3) & ~(size_t)3;                 // 16-byte alignment for Cand
    words += 4 * (size_t)C + 2 * (size_t)K;
    words = (words + 3) & ~(size_t)3;
    const size_t per_warp = words * 4;
    int wpb = (int)((96 * 1024) / per_warp);
    if (wpb > 8) wpb = 8;
    if (wpb < 1) wpb = 1;
    const size_t smem = per_warp * wpb;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(merge_topk_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    const unsigned grid = (unsigned)((L + wpb - 1) / wpb);
    merge_topk_kernel<<<grid, 32 * wpb, smem, st>>>(row_val, row_idx, col_val, col_idx, L, N_c, K,
                                                    Kr, Kc, C, words, idx, score, gate);
    return cudaGetLastError();
}

}  // namespace omni

// shared_mlp.cu -- the shared dense MLP that the layer adds to the routed
// branch, on the sm_100a tensor cores.
//
// "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale"
// (rainbus review page, method paragraph, step 1: the layer's output is the
// routed assembly plus MLP(x); gist.science summary (German edition),
// section 2.1 "Kernkomponenten": a standard dense MLP branch is active for
// every input).  The pages give the MLP no form; it is taken as the gated one,
//     h = SiLU(x W_g^T) * (x W_u^T)   (rounded to bf16, the operand type of
//                                       the second product)
//     y (+)= h W_d^T
// with W_g, W_u stored as F rows of d and W_d as d rows of F (all K-major).
//
// One persistent tile GEMM, launched twice.  Tiles are 128 x 256 with a K
// step of 64; warp 0 issues TMA loads (each CTA its own) into a 4-stage ring,
// warp 1 issues tcgen05.mma kind::f16 into one of two 256-column TMEM
// accumulators (all 512 columns), warps 2-9 drain the other one.
//   up:   the B tile is 128 rows of W_g stacked on the same 128 rows of W_u,
//         so accumulator columns 0-127 are gate pre-activations and 128-255
//         the matching up projections; the epilogue writes h for those 128
//         hidden units.
//   down: A = h, the B tile is 256 rows of W_d; the epilogue adds the fp32
//         tile into y (or stores it).  Every y element belongs to one tile,
//         so there are no atomics and the sum has a fixed order.
// Rows past L, F or d read as zeros through TMA out-of-bounds fill and are
// masked on store; a second B box that starts past the end is not loaded
// (its accumulator columns are never stored).
#include <cuda_bf16.h>

#include "omni_common.cuh"
#include "omni_internal.h"
#include "tcgen05.cuh"

namespace omni {
namespace {

constexpr int BM = 128, BN = 256, BK = kSwK, STAGES = 4;
constexpr int kBoxRows = BN / 2;                 // rows of one B box
constexpr int kTileBytesA = BM * BK * 2;         // 16 KB
constexpr int kBoxBytesB = kBoxRows * BK * 2;    // 16 KB
constexpr int kTileBytesB = 2 * kBoxBytesB;      // 32 KB
constexpr uint32_t kTmemCols = 2 * BN;           // two fp32 accumulators
constexpr int kEpiWarps = 8;                     // two per TMEM lane quarter, half the columns each
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr uint32_t kIdesc = umma_idesc_bf16(BM, BN);

enum : int { kEpiUp = 0, kEpiDown = 1 };

struct __align__(1024) MlpSmem {
    uint8_t a[STAGES][kTileBytesA];
    uint8_t b[STAGES][kTileBytesB];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];                           // accumulator ready for the epilogue
    uint64_t tempty[2];                          // accumulator drained
    uint32_t tmem_base;
    int abort;
};

struct MlpPass {
    int M;            // rows of A (tokens)
    int K;            // contraction length (d, then F)
    int ntn;          // n tiles
    int b_rows;       // rows of the B tensors (F, then d)
    int b_step;       // B rows per n tile: 128 (up) or 256 (down)
    int b1_off;       // row offset of the second B box: 0 (up: W_u) or 128 (down)
    int n_out;        // output columns: F (h) or d (y)
    uint16_t *h;      // up: [M, F] bf16
    float *y;         // down: [M, d] fp32
    int accumulate;   // down: y += tile
    int *status;
};

__device__ __forceinline__ float silu_f32(float z) { return z / (1.f + __expf(-z)); }

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
mlp_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                const __grid_constant__ CUtensorMap tm_b1, const MlpPass p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment of the tiles is required by the swizzled layout
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    MlpSmem &sm = *reinterpret_cast<MlpSmem *>(smem_raw + pad);
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    const int nk = (p.K + BK - 1) / BK;
    const int ntiles = ((p.M + BM - 1) / BM) * p.ntn;
    int *status = p.status;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.tfull[b], 1);
            mbar_init(&sm.tempty[b], kEpiWarps);
        }
        sm.abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&sm.tmem_base)), "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // everything above touches only this CTA's shared memory and TMEM
    grid_dependency_wait();
    grid_dependents_launch();

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer
            int it = 0, issued_from = 0;
            for (int tile = blockIdx.x; tile < ntiles && !sm.abort; tile += gridDim.x) {
                const int m0 = (tile / p.ntn) * BM;
                const int r0 = (tile % p.ntn) * p.b_step;
                const int r1 = r0 + p.b1_off;
                const bool second = r1 < p.b_rows;
                const uint32_t bytes = kTileBytesA + (second ? 2 : 1) * kBoxBytesB;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (it >= STAGES &&
                        !mbar_wait(&sm.empty[s], (uint32_t)(((it / STAGES) - 1) & 1), status)) {
                        sm.abort = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.full[s], bytes);
                    tma_load_2d(sm.a[s], &tm_a, kb * BK, m0, &sm.full[s]);
                    tma_load_2d(sm.b[s], &tm_b0, kb * BK, r0, &sm.full[s]);
                    if (second) tma_load_2d(sm.b[s] + kBoxBytesB, &tm_b1, kb * BK, r1, &sm.full[s]);
                    issued_from = it + 1 > STAGES ? it + 1 - STAGES : 0;
                }
            }
            if (sm.abort) {
                // let the loads already issued land before the CTA can exit
                for (int k = issued_from; k < it; ++k)
                    mbar_wait(&sm.full[k % STAGES], (uint32_t)((k / STAGES) & 1), status);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer
            int it = 0, lt = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++lt) {
                const int buf = lt & 1;
                if (lt >= 2 && !mbar_wait(&sm.tempty[buf], (uint32_t)(((lt >> 1) - 1) & 1), status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(buf * BN);
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (!mbar_wait(&sm.full[s], (uint32_t)((it / STAGES) & 1), status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(sm.a[s]);
                    const uint64_t bd = sw128_desc(sm.b[s]);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        // advance 16 bf16 = 32 bytes along K inside the swizzle atom
                        umma_bf16(acc, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), kIdesc,
                                  (kb > 0 || k > 0) ? 1u : 0u);
                    }
                    umma_commit(&sm.empty[s]);
                }
                umma_commit(&sm.tfull[buf]);      // arrives once this tile's MMAs are done
            }
            if (!ok) sm.abort = 1;
        }
        __syncwarp();
    } else {
        // ---- epilogue: warp w reads TMEM lanes 32*(w % 4) .. +31 (tile rows)
        const int quarter = warp & 3;
        const int half = (warp - 2) >> 2;
        int lt = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++lt) {
            const int buf = lt & 1;
            if (!mbar_wait(&sm.tfull[buf], (uint32_t)((lt >> 1) & 1), status)) break;
            tc_fence_after();
            const int m0 = (tile / p.ntn) * BM;
            const int tn = tile % p.ntn;
            const int row = m0 + quarter * 32 + (int)lane;
            const uint32_t tb = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
            if (EPI == kEpiUp) {
                // this warp: hidden units f0 .. f0 + 63 (gate at column u, up at u + 128)
                const int u0 = half * 64;
                const int f0 = tn * kBoxRows + u0;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t g[32], v[32];
                    tmem_ld32(tb + (uint32_t)(u0 + 32 * c), g);
                    tmem_ld32(tb + (uint32_t)(kBoxRows + u0 + 32 * c), v);
                    const int f = f0 + 32 * c;
                    if (row < p.M && f < p.n_out) {
                        uint32_t hp[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float lo = silu_f32(__uint_as_float(g[2 * j])) * __uint_as_float(v[2 * j]);
                            const float hi =
                                silu_f32(__uint_as_float(g[2 * j + 1])) * __uint_as_float(v[2 * j + 1]);
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(lo, hi);
                            hp[j] = *reinterpret_cast<const uint32_t *>(&b2);
                        }
                        uint4 *dst = reinterpret_cast<uint4 *>(p.h + (size_t)row * p.n_out + f);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(hp[4 * q], hp[4 * q + 1], hp[4 * q + 2], hp[4 * q + 3]);
                    }
                }
            } else {
                // this warp: output columns n0 .. n0 + 127
                const int n0 = tn * BN + half * kBoxRows;
#pragma unroll
                for (int c = 0; c < kBoxRows / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tb + (uint32_t)(half * kBoxRows + 32 * c), r);
                    const int col = n0 + 32 * c;
                    if (row < p.M && col < p.n_out) {
                        float4 *dst = reinterpret_cast<float4 *>(p.y + (size_t)row * p.n_out + col);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            float4 o = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                                   __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
                            if (p.accumulate) {
                                const float4 prev = dst[q];
                                o.x += prev.x;
                                o.y += prev.y;
                                o.z += prev.z;
                                o.w += prev.w;
                            }
                            dst[q] = o;
                        }
                    }
                }
            }
            // this accumulator may be overwritten once every epilogue warp is done
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.tempty[buf]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem), "r"(kTmemCols));
    }
}

template <int EPI>
cudaError_t launch_pass(const CUtensorMap &a, const CUtensorMap &b0, const CUtensorMap &b1,
                        const MlpPass &p, cudaStream_t st) {
    const int smem = (int)sizeof(MlpSmem) + 1024;   // slack for base alignment
    const cudaError_t e = cudaFuncSetAttribute(mlp_gemm_kernel<EPI>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int ntiles = ((p.M + BM - 1) / BM) * p.ntn;
    const int sms = device_sm_count();
    const int grid = ntiles < sms ? ntiles : sms;
    return launch(mlp_gemm_kernel<EPI>, dim3(grid), dim3(kThreads), (size_t)smem, st, a, b0, b1, p);
}

}  // namespace

cudaError_t launch_shared_mlp(const uint16_t *x, const uint16_t *W_g, const uint16_t *W_u,
                              const uint16_t *W_d, int L, int d, int F, uint16_t *h, float *y,
                              bool accumulate, int *status, cudaStream_t st) {
    CUtensorMap tm_x, tm_g, tm_u, tm_h, tm_d;
    if (!make_sw128_map(&tm_x, x, L, d, BM) || !make_sw128_map(&tm_g, W_g, F, d, kBoxRows) ||
        !make_sw128_map(&tm_u, W_u, F, d, kBoxRows) || !make_sw128_map(&tm_h, h, L, F, BM) ||
        !make_sw128_map(&tm_d, W_d, d, F, kBoxRows))
        return cudaErrorInvalidValue;
    MlpPass up;
    up.M = L; up.K = d; up.ntn = (F + kBoxRows - 1) / kBoxRows; up.b_rows = F;
    up.b_step = kBoxRows; up.b1_off = 0; up.n_out = F; up.h = h; up.y = nullptr;
    up.accumulate = 0; up.status = status;
    MlpPass down;
    down.M = L; down.K = F; down.ntn = (d + BN - 1) / BN; down.b_rows = d;
    down.b_step = BN; down.b1_off = kBoxRows; down.n_out = d; down.h = nullptr; down.y = y;
    down.accumulate = accumulate ? 1 : 0; down.status = status;
    cudaError_t e = launch_pass<kEpiUp>(tm_x, tm_g, tm_u, up, st);
    if (e != cudaSuccess) return e;
    return launch_pass<kEpiDown>(tm_h, tm_d, tm_d, down, st);
}

}  // namespace omni

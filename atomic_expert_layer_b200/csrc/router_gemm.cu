// router_gemm.cu -- router projections on the sm_100a tensor cores.
//
// "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale"
// (rainbus review page, method paragraph, step 2; gist.science summary,
// section 2.2 "Kartesischer Produkt-Router"): s_r = x W_r and s_c = x W_c,
// two d x sqrt(N) projections instead of one d x N.  W_r / W_c are stored as
// N_r / N_c rows of d, so both operands are K-major.
//
// One persistent launch computes both, K step 64 (one 128-byte swizzle atom
// of bf16).  Warp roles: warp 0 issues TMA tile loads into a 6-stage
// shared-memory ring; warp 1 of the pair's first CTA issues tcgen05.mma
// kind::f16 (bf16 in, fp32 accumulate) into one of two TMEM accumulators;
// warps 2-9 drain the other accumulator with tcgen05.ld (two warps per TMEM
// lane quarter, one per column half), write the fp32 logits and, per (token,
// tile, half), the maximum and the sum of exp(s - max) over those columns --
// the LogSoftmax partials -- so the epilogue of one tile overlaps the main
// loop of the next.  Ragged edges (L,
// N_r, N_c, d not multiples of the tile) read as zeros through TMA
// out-of-bounds fill and are masked on store.
#include "omni_common.cuh"
#include "omni_internal.h"
#include "router_small.cuh"
#include "tcgen05.cuh"

namespace omni {
namespace {

// Tiles are 256 x 224 (n-tiles of W_r first, then those of W_c), computed by
// a pair of CTAs (a cluster of 2, tcgen05.mma.cta_group::2): CTA r of the
// pair loads rows m0 + 128 r .. + 127 of x and rows n0 + 112 r .. + 111 of
// the W tile into its own shared memory, the pair's first CTA issues the
// MMAs, and each CTA's TMEM receives its 128 rows of the 256 x 224 product.
// Per output element this moves about half the operand bytes of a one-CTA
// 128 x 128 tile, and 224 columns pad a 1304-wide axis by 3% (6 tiles).
constexpr int BM = 128;                      // rows per CTA (256 per pair)
constexpr int BN = 224;                      // columns per tile
constexpr int BNH = BN / 2;                  // W rows per CTA per tile
constexpr int BK = kSwK, STAGES = 6;
constexpr int kTileBytesA = BM * BK * 2;     // 16 KB
constexpr int kTileBytesB = BNH * BK * 2;    // 14 KB
constexpr int kAccStride = 256;              // TMEM columns between the two accumulators
constexpr uint32_t kTmemCols = 512;
constexpr int kEpiWarps = 8;                 // two per TMEM lane quarter
constexpr int kThreads = 32 * (2 + kEpiWarps);  // producer, MMA, epilogue warps
constexpr int kChunksHalf0 = 4;              // 32-column chunks of epilogue half 0 (then 3)
static_assert(2 * kGemmPartCols == BN, "two LogSoftmax partials per tile");

struct __align__(1024) GemmSmem {
    uint8_t a[STAGES][kTileBytesA];
    uint8_t b[STAGES][kTileBytesB];
    float stage[kEpiWarps][32 * 32];         // per epilogue warp: a 32 x 32 block for the TMA store
    uint64_t full[STAGES];                   // used in the pair's first CTA
    uint64_t empty[STAGES];
    uint64_t tfull[2];                       // accumulator ready for the epilogue
    uint64_t tempty[2];                      // accumulator drained (first CTA: both CTAs' warps)
    uint32_t tmem_base;
    int abort;
};

constexpr uint32_t kIdesc = umma_idesc_bf16(2 * BM, BN);

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
router_gemm_kernel(const __grid_constant__ CUtensorMap tm_x,
                   const __grid_constant__ CUtensorMap tm_wr,
                   const __grid_constant__ CUtensorMap tm_wc,
                   const __grid_constant__ CUtensorMap tm_sr,
                   const __grid_constant__ CUtensorMap tm_sc, int store_r, int store_c,
                   float *__restrict__ s_r,
                   float *__restrict__ s_c, float2 *__restrict__ part_r,
                   float2 *__restrict__ part_c, int L, int d, int N_r, int N_c, int ntile_r,
                   int ntile_c, int *status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment of the tiles is required by the swizzled layout
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    GemmSmem &sm = *reinterpret_cast<GemmSmem *>(smem_raw + pad);
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    const uint32_t rank = cluster_ctarank();         // 0: issues the MMAs
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int nk = (d + BK - 1) / BK;
    const int nnt = ntile_r + ntile_c;
    const int ntiles = ((L + 2 * BM - 1) / (2 * BM)) * nnt;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.tfull[b], 1);
            mbar_init(&sm.tempty[b], 2 * kEpiWarps);
        }
        sm.abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&sm.tmem_base)), "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                                  // both CTAs' barriers exist
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // everything above touches only the pair's shared memory and TMEM
    grid_dependency_wait();
    grid_dependents_launch();

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer (both CTAs): completion counted on the first CTA's barrier
            int it = 0, issued_from = 0;
            for (int tile = pair; tile < ntiles && !sm.abort; tile += npairs) {
                const int m0 = (tile / nnt) * (2 * BM) + (int)rank * BM;
                const int nt = tile % nnt;
                const bool col_axis = nt >= ntile_r;
                const int n0 = (col_axis ? nt - ntile_r : nt) * BN + (int)rank * BNH;
                const CUtensorMap *tm_b = col_axis ? &tm_wc : &tm_wr;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (it >= STAGES &&
                        !mbar_wait(&sm.empty[s], (uint32_t)(((it / STAGES) - 1) & 1), status)) {
                        sm.abort = 1;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&sm.full[s], 2 * (kTileBytesA + kTileBytesB));
                    const uint32_t fb = smem_in_cta(&sm.full[s], 0);
                    tma_load_2d_pair(sm.a[s], &tm_x, kb * BK, m0, fb);
                    tma_load_2d_pair(sm.b[s], tm_b, kb * BK, n0, fb);
                    issued_from = it + 1 > STAGES ? it + 1 - STAGES : 0;
                }
            }
            if (sm.abort && rank == 0) {
                // let the loads already issued land before the CTA can exit
                for (int k = issued_from; k < it; ++k)
                    mbar_wait_cluster(&sm.full[k % STAGES], (uint32_t)((k / STAGES) & 1), status);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---- MMA issuer (the pair's first CTA)
            int it = 0, lt = 0;
            bool ok = true;
            for (int tile = pair; tile < ntiles && ok; tile += npairs, ++lt) {
                const int buf = lt & 1;
                if (lt >= 2 &&
                    !mbar_wait_cluster(&sm.tempty[buf], (uint32_t)(((lt >> 1) - 1) & 1), status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(buf * kAccStride);
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (!mbar_wait_cluster(&sm.full[s], (uint32_t)((it / STAGES) & 1), status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(sm.a[s]);
                    const uint64_t bd = sw128_desc(sm.b[s]);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        // advance 16 bf16 = 32 bytes along K inside the swizzle atom
                        umma_bf16_pair(acc, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), kIdesc,
                                       (kb > 0 || k > 0) ? 1u : 0u);
                    }
                    umma_commit_pair(&sm.empty[s]);    // frees stage s in both CTAs
                }
                umma_commit_pair(&sm.tfull[buf]);      // both CTAs' epilogues may read
            }
            if (!ok) sm.abort = 1;
        }
        __syncwarp();
    } else {
        // ---- epilogue: warp w reads TMEM lanes 32*(w % 4) .. +31 (this CTA's
        // rows of the tile); half 0 takes columns 0-127, half 1 columns 128-223
        const int quarter = warp & 3;
        const int half = (warp - 2) >> 2;
        const int c_lo = half == 0 ? 0 : kChunksHalf0;
        const int c_hi = half == 0 ? kChunksHalf0 : BN / 32;
        const uint32_t tempty0 = smem_in_cta(&sm.tempty[0], 0);
        const uint32_t tempty1 = smem_in_cta(&sm.tempty[1], 0);
        float *stage = sm.stage[warp - 2];
        int lt = 0;
        for (int tile = pair; tile < ntiles; tile += npairs, ++lt) {
            const int buf = lt & 1;
            if (!mbar_wait(&sm.tfull[buf], (uint32_t)((lt >> 1) & 1), status)) break;
            tc_fence_after();
            const int m0 = (tile / nnt) * (2 * BM) + (int)rank * BM;
            const int nt = tile % nnt;
            const bool col_axis = nt >= ntile_r;
            const int tn = col_axis ? nt - ntile_r : nt;
            const int n_axis = col_axis ? N_c : N_r;
            const int row0 = m0 + quarter * 32;
            const int row = row0 + (int)lane;
            float *out = (col_axis ? s_c : s_r) + (size_t)row * n_axis;
            const bool vec = (n_axis & 3) == 0;
            // whole-line writes: the warp's 32 x 32 block goes out as one TMA
            // store from 128-byte-swizzled shared memory (rows of 16-byte
            // multiples only; otherwise each thread stores its row)
            const bool by_tma = col_axis ? store_c != 0 : store_r != 0;
            const CUtensorMap *tm_s = col_axis ? &tm_sc : &tm_sr;
            float M = -INFINITY, S = 0.f;
            for (int c = c_lo; c < c_hi; ++c) {
                uint32_t r[32];
                tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) +
                              (uint32_t)(buf * kAccStride + c * 32), r);
                const int col = tn * BN + c * 32;
                float mx = -INFINITY, sm_ = 0.f;
                if (col + 32 <= n_axis) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) mx = fmaxf(mx, __uint_as_float(r[j]));
#pragma unroll
                    for (int j = 0; j < 32; ++j) sm_ += __expf(__uint_as_float(r[j]) - mx);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (col + j < n_axis) mx = fmaxf(mx, __uint_as_float(r[j]));
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (col + j < n_axis) sm_ += __expf(__uint_as_float(r[j]) - mx);
                }
                // fold this chunk's (max, sum) into the half's running pair
                if (mx > -INFINITY) {
                    const float nm = fmaxf(M, mx);
                    S = (M > -INFINITY ? S * __expf(M - nm) : 0.f) + sm_ * __expf(mx - nm);
                    M = nm;
                }
                if (by_tma) {
                    if (lane == 0) bulk_wait_read0();        // the previous block has left
                    __syncwarp();
                    float4 *st4 = reinterpret_cast<float4 *>(stage + lane * 32);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        st4[j ^ (int)(lane & 7u)] =
                            make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                        __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && row0 < L && col < n_axis) {
                        tma_store_2d(tm_s, col, row0, stage);
                        bulk_commit();
                    }
                } else if (row < L) {
                    if (vec && col + 32 <= n_axis) {
                        float4 *o4 = reinterpret_cast<float4 *>(out + col);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            o4[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                                __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (col + j < n_axis) out[col + j] = __uint_as_float(r[j]);
                    }
                }
            }
            // this accumulator may be overwritten once every epilogue warp of
            // both CTAs is done (the first CTA's barrier counts all 16)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(buf ? tempty1 : tempty0);
            if (row < L) {
                // one (max, sum) pair per (row, tile, column half); a half with
                // no valid column gives (-inf, 0)
                float2 *part = col_axis ? part_c : part_r;
                const int nta = col_axis ? ntile_c : ntile_r;
                part[((size_t)row * nta + tn) * 2 + half] = make_float2(M, S);
            }
        }
    }
    if (warp >= 2 && lane == 0) bulk_wait_read0();   // shared memory outlives the stores' reads
    tc_fence_before();
    __syncthreads();
    cluster_sync();                                  // the pair is done with both TMEMs
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem), "r"(kTmemCols));
    }
}

template <int LM>
__global__ void __launch_bounds__(32 * kSmallWarps)
router_small_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ W_r,
                    const uint16_t *__restrict__ W_c, int L, int d, int N_r, int N_c,
                    float *__restrict__ s_r, float *__restrict__ s_c) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint4 *xs = reinterpret_cast<uint4 *>(smem);      // [L][d / 8]
    grid_dependency_wait();
    grid_dependents_launch();
    const int d8 = d >> 3;
    const int warp = threadIdx.x >> 5;
    const int g0 = (blockIdx.x * kSmallWarps + warp) * kSmallRows;
    small_rows_dot<LM>(xs, W_r, W_c, L, d, N_r, N_c, g0, s_r, s_c, [&]() {
        // x rows into shared memory, every copy in flight at once
        for (int i = threadIdx.x; i < L * d8; i += blockDim.x)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                         ::"r"(smem_u32(xs + i)), "l"(reinterpret_cast<const uint4 *>(x) + i)
                         : "memory");
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
    });
}

template <int LM>
cudaError_t launch_small_lm(const uint16_t *x, const uint16_t *W_r, const uint16_t *W_c, int L,
                            int d, int N_r, int N_c, float *s_r, float *s_c, cudaStream_t st) {
    const size_t smem = (size_t)L * d * 2;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(
            router_small_kernel<LM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int rows_per_cta = kSmallWarps * kSmallRows;
    const unsigned grid = (unsigned)((N_r + N_c + rows_per_cta - 1) / rows_per_cta);
    return launch(router_small_kernel<LM>, dim3(grid), dim3(32 * kSmallWarps), smem, st, x, W_r,
                  W_c, L, d, N_r, N_c, s_r, s_c);
}

}  // namespace

cudaError_t launch_router_gemm(const uint16_t *x, const uint16_t *W_r, const uint16_t *W_c,
                               int L, int d, int N_r, int N_c, float *s_r, float *s_c,
                               float *part_r, float *part_c, int *status, cudaStream_t st) {
    CUtensorMap tm_x, tm_wr, tm_wc, tm_sr, tm_sc;
    if (!make_sw128_map(&tm_x, x, L, d, BM) || !make_sw128_map(&tm_wr, W_r, N_r, d, BNH) ||
        !make_sw128_map(&tm_wc, W_c, N_c, d, BNH))
        return cudaErrorInvalidValue;
    // TMA stores of the logits need 16-byte rows and a 16-byte-aligned base
    const bool al_r = (reinterpret_cast<uintptr_t>(s_r) & 15u) == 0;
    const bool al_c = (reinterpret_cast<uintptr_t>(s_c) & 15u) == 0;
    const int store_r = al_r && N_r % 4 == 0 && make_f32_store_map(&tm_sr, s_r, L, N_r) ? 1 : 0;
    const int store_c = al_c && N_c % 4 == 0 && make_f32_store_map(&tm_sc, s_c, L, N_c) ? 1 : 0;
    if (!store_r) tm_sr = tm_x;                        // unused
    if (!store_c) tm_sc = tm_x;
    const int smem = (int)sizeof(GemmSmem) + 1024;   // slack for base alignment
    cudaError_t e = cudaFuncSetAttribute(router_gemm_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int ntile_r = (N_r + BN - 1) / BN, ntile_c = (N_c + BN - 1) / BN;
    const int ntiles = ((L + 2 * BM - 1) / (2 * BM)) * (ntile_r + ntile_c);
    const int pairs_max = device_sm_count() / 2;
    const int pairs = ntiles < pairs_max ? ntiles : pairs_max;
    return launch(router_gemm_kernel, dim3(2 * pairs), dim3(kThreads), (size_t)smem, st, tm_x,
                  tm_wr, tm_wc, tm_sr, tm_sc, store_r, store_c, s_r, s_c,
                  reinterpret_cast<float2 *>(part_r),
                  reinterpret_cast<float2 *>(part_c), L, d, N_r, N_c, ntile_r, ntile_c, status);
}

}  // namespace omni

namespace omni {

bool router_small_ok(int L, int d) { return L <= 4 && d <= 32 * 8 * kSmallSlices; }

cudaError_t launch_router_small(const uint16_t *x, const uint16_t *W_r, const uint16_t *W_c,
                                int L, int d, int N_r, int N_c, float *s_r, float *s_c,
                                cudaStream_t st) {
    if (L <= 1) return launch_small_lm<1>(x, W_r, W_c, L, d, N_r, N_c, s_r, s_c, st);
    if (L <= 2) return launch_small_lm<2>(x, W_r, W_c, L, d, N_r, N_c, s_r, s_c, st);
    if (L <= 4) return launch_small_lm<4>(x, W_r, W_c, L, d, N_r, N_c, s_r, s_c, st);
    if (L <= 8) return launch_small_lm<8>(x, W_r, W_c, L, d, N_r, N_c, s_r, s_c, st);
    return launch_small_lm<16>(x, W_r, W_c, L, d, N_r, N_c, s_r, s_c, st);
}

}  // namespace omni

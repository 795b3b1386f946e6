// expert_dense.cu -- the grouped expert computation on the sm_100a tensor
// cores, for the experts that many tokens share.
//
// "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale"
// (rainbus review page, method paragraph, step 3; gist.science summary,
// section 2.2 "Experten-zentriertes Scheduling"): every active group q runs a
// grouped GEMM
//     O_q = (G_q . SiLU(X_q W_q^T)) V_q,        y[t] += O_q[t],
// with G_q the gate of each (token, expert) task of the group and 0 elsewhere.
//
// G_q is dense enough for the tensor cores only in the columns of experts that
// many tokens route to.  Here an expert is "dense" when at least `thr` tasks
// use it (the threshold grows with the batch: the tile GEMM spends 4 L d
// flops per dense expert, the task-by-task path a row gather per task); the
// group's other tasks stay on the task-by-task CUDA-core path (expert.cu).
// The dense experts of all active groups, in group order, are laid side by
// side as the N columns of one product over all L tokens:
//     H = X W_D^T                     [L, E] on the tensor cores (fp32 in TMEM)
//     P = G . SiLU(H)                 in the epilogue, rounded to bf16
//     y += P V_D                      [L, d] on the tensor cores
// The columns of group q are its block of the grouped GEMM; a token that has
// no task on a column has a zero gate there, so the zero rows of G_q cost
// flops but change nothing.  The sum over groups of y[t] += O_q[t] happens in
// the TMEM accumulator of the second product, whose K dimension runs over the
// dense experts of every group, so y is written once per element (no atomics).
//
// Steps (all on the caller's stream, no host synchronisation, no spin-waits):
//   1. count:   tasks per expert over the whole list; then per active group
//               the number of its experts with >= thr tasks.
//   2. scan:    exclusive scan of the per-group counts -> each group's first
//               dense column; the total is E (capped at `cap` columns).
//   3. list:    per group, the ids of its dense experts in column order; each
//               one's counter becomes -(column + 1).  Experts past the cap get
//               no column and stay task by task.
//   4. gather:  W_D = the dense experts' W rows [cap, d] and V_D^T [d, cap]
//               (zero past E), and G zeroed over the E_pad columns in use.
//   5. split:   each task either writes its gate into G (dense expert) or is
//               appended to the compacted list of the CUDA-core path.
//   6. (expert.cu) the CUDA-core passes on the compacted tasks write y.
//   7. gemm 1:  P = G . SiLU(X W_D^T), 128 x 256 tiles, TMA-fed tcgen05.mma.
//   8. gemm 2:  y += P V_D, 128 x 256 tiles, TMA-fed tcgen05.mma.
// Both GEMMs read the number of dense experts from the workspace, so the
// host never waits for it.
#include <cuda_bf16.h>

#include "omni_common.cuh"
#include "omni_internal.h"
#include "tcgen05.cuh"

namespace omni {
namespace {

// ---------------------------------------------------------------- 1. count
// (a) Tasks per expert over the whole sorted list (grid-stride, 32
// consecutive tasks per warp; equal experts inside a warp are added by one
// atomic).  Checks that every task lies in its group's range of the sorted
// order (group_offsets).
__global__ void __launch_bounds__(256)
dense_use_kernel(const int32_t *__restrict__ task_expert, int64_t M,
                 const int32_t *__restrict__ off, int B, int64_t N, int32_t *__restrict__ cnt,
                 int *status) {
    grid_dependency_wait();
    grid_dependents_launch();
    const unsigned lane = lane_id();
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t base = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 32;
         base < M; base += nwarps * 32) {
        const int64_t m = base + lane;
        int32_t key = -1;
        if (m < M) {
            const int32_t e = task_expert[m];
            bool ok = e >= 0 && (int64_t)e < N;
            if (ok) {
                const int64_t q = e / B;
                ok = m >= off[q] && m < off[q + 1];
            }
            if (ok)
                key = e;
            else
                set_status(status, OMNI_DEV_BAD_SCHEDULE);
        }
        const unsigned peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && lane == (unsigned)(__ffs(peers) - 1)) atomicAdd(&cnt[key], __popc(peers));
    }
}

// (b) Warp per active group: the number of its experts with >= thr tasks.
// Checks num_active, the group ids and their offsets, and adds up the
// tasks the active groups cover (the split step checks that it is M).
__global__ void dense_mark_kernel(const int32_t *__restrict__ cnt, const int32_t *__restrict__ off,
                                  const int32_t *__restrict__ active,
                                  const int32_t *__restrict__ num_active, int64_t G, int B,
                                  int64_t N, int64_t M, int thr, int32_t *__restrict__ ghot,
                                  int32_t *__restrict__ covered, int *status) {
    grid_dependency_wait();
    grid_dependents_launch();
    const unsigned lane = lane_id();
    const int gwarp = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    int nact = *num_active;
    if (nact < 0 || (int64_t)nact > G) {
        if (gwarp == 0 && lane == 0) set_status(status, OMNI_DEV_BAD_SCHEDULE);
        nact = nact < 0 ? 0 : (int)G;
    }
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    for (int i = gwarp; i < nact; i += nwarps) {
        const int32_t q = active[i];
        if (q < 0 || (int64_t)q >= G) {
            if (lane == 0) set_status(status, OMNI_DEV_BAD_SCHEDULE);
            continue;
        }
        const int32_t o0 = off[q], o1 = off[q + 1];
        if (o0 < 0 || (int64_t)o1 > M || o1 < o0) {
            if (lane == 0) set_status(status, OMNI_DEV_BAD_SCHEDULE);
            continue;
        }
        if (lane == 0) atomicAdd(covered, o1 - o0);
        if (o1 - o0 < thr) continue;                  // no expert of q can reach thr
        const int64_t base = (int64_t)q * B;
        int nh = 0;
        for (int j0 = 0; j0 < B; j0 += 32) {
            const int j = j0 + (int)lane;
            const int64_t e = base + j;
            nh += __popc(__ballot_sync(0xffffffffu, j < B && e < N && cnt[e] >= thr));
        }
        if (lane == 0) ghot[q] = nh;
    }
}

// ----------------------------------------------------------------- 3. list
// Warp per active group with dense experts: their ids in column order, and
// each one's counter replaced by -(column + 1), which is how the split step
// tells a dense expert and finds its column.  Columns at or past `cap` are not
// built; those experts keep their (positive) counts and stay on the CUDA-core
// path.  They are the highest columns (the last ones of a group, and every
// later group), so the columns of the others do not move.
__global__ void dense_list_kernel(const int32_t *__restrict__ hoff,
                                  const int32_t *__restrict__ active,
                                  const int32_t *__restrict__ num_active, int64_t G, int B,
                                  int64_t N, int thr, int cap, int32_t *__restrict__ cnt,
                                  int32_t *__restrict__ list) {
    grid_dependency_wait();
    grid_dependents_launch();
    const unsigned lane = lane_id();
    int nact = *num_active;
    nact = nact < 0 ? 0 : ((int64_t)nact > G ? (int)G : nact);
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    for (int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < nact; i += nwarps) {
        const int32_t q = active[i];
        if (q < 0 || (int64_t)q >= G) continue;
        const int32_t h0 = hoff[q];
        if (hoff[q + 1] == h0) continue;
        const int64_t base = (int64_t)q * B;
        int run = 0;
        for (int j0 = 0; j0 < B; j0 += 32) {
            const int j = j0 + (int)lane;
            const int64_t e = base + j;
            const bool hot = j < B && e < N && cnt[e] >= thr;
            const unsigned bal = __ballot_sync(0xffffffffu, hot);
            const int h = h0 + run + __popc(bal & lanemask_lt());
            if (hot && h < cap) {
                list[h] = (int32_t)e;
                cnt[e] = -(h + 1);
            }
            run += __popc(bal);
        }
    }
}

__device__ __forceinline__ int dense_count(const int32_t *ehot, int cap) {
    const int e = *ehot;
    return e < cap ? e : cap;
}

// --------------------------------------------------------------- 4. gather
// W_D rows and V_D^T columns of the dense experts (zero past E, up to the
// next multiple of 256), and G zeroed over those columns for every token.
constexpr int kGatherThreads = 256;
constexpr int kTp = 72;                    // shared row pitch (bf16) of a 64 x 64 tile

__global__ void __launch_bounds__(kGatherThreads)
dense_gather_kernel(const uint16_t *__restrict__ W, const uint16_t *__restrict__ V, int d,
                    int L, int64_t N, const int32_t *__restrict__ list,
                    const int32_t *__restrict__ ehot, int cap, uint16_t *__restrict__ whot,
                    uint16_t *__restrict__ vt, float *__restrict__ Gm) {
    __shared__ __align__(16) uint16_t tile[64 * kTp];
    grid_dependency_wait();
    grid_dependents_launch();
    const int tid = threadIdx.x;
    const int E = dense_count(ehot, cap);
    const int Ep = (E + 255) & ~255;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    // expert of column h, or -1 past E (an id out of range reads as zeros)
    auto expert_of = [&](int h) -> int64_t {
        if (h >= E) return -1;
        const int64_t e = list[h];
        return e >= 0 && e < N ? e : -1;
    };
    // W_D: one row per iteration
    for (int r = blockIdx.x; r < Ep; r += gridDim.x) {
        const int64_t er = expert_of(r);
        const uint4 *src = er >= 0 ? reinterpret_cast<const uint4 *>(W + (size_t)er * d) : nullptr;
        uint4 *dst = reinterpret_cast<uint4 *>(whot + (size_t)r * d);
        for (int c = tid; c < d / 8; c += kGatherThreads) dst[c] = src ? src[c] : zero;
    }
    // V_D^T: 64 experts x 64 features per tile, transposed through shared memory
    const int nth = Ep / 64, ntd = d / 64;
    for (int tl = blockIdx.x; tl < nth * ntd; tl += gridDim.x) {
        const int hb = tl % nth, db = tl / nth;
        for (int k = tid; k < 64 * 8; k += kGatherThreads) {
            const int rr = k >> 3, seg = k & 7;
            const int64_t eh = expert_of(hb * 64 + rr);
            const uint4 v = eh >= 0 ? *reinterpret_cast<const uint4 *>(V + (size_t)eh * d +
                                                                       db * 64 + seg * 8)
                                    : zero;
            *reinterpret_cast<uint4 *>(&tile[rr * kTp + seg * 8]) = v;
        }
        __syncthreads();
        for (int k = tid; k < 64 * 8; k += kGatherThreads) {
            const int dd = k >> 3, seg = k & 7;
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                w[u] = (uint32_t)tile[(seg * 8 + 2 * u) * kTp + dd] |
                       ((uint32_t)tile[(seg * 8 + 2 * u + 1) * kTp + dd] << 16);
            *reinterpret_cast<uint4 *>(vt + (size_t)(db * 64 + dd) * cap + hb * 64 + seg * 8) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
        __syncthreads();
    }
    // G over columns [0, Ep)
    const int q4 = Ep / 4;
    const int64_t total = (int64_t)L * q4;
    const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t i = (int64_t)blockIdx.x * kGatherThreads + tid; i < total;
         i += (int64_t)gridDim.x * kGatherThreads) {
        const int64_t t = i / q4;
        const int c = (int)(i - t * q4);
        reinterpret_cast<float4 *>(Gm + (size_t)t * cap)[c] = z4;
    }
}

// ---------------------------------------------------------------- 5. split
// Each warp takes chunks of 32 x 32 tasks.  A task whose expert has a
// column (counter < 0) writes its gate into G at (token, column); the other
// tasks are appended, in chunk order, to the compacted list of the CUDA-core
// path: lane r keeps the ballot of round r, the warp reserves the chunk's
// room with one atomic and re-reads only the tasks it appends.  Also checks
// that the active groups cover all M tasks (num_active too small, or an
// active group missing or listed twice).
constexpr int kSplitRounds = 32;

__global__ void __launch_bounds__(256)
dense_split_kernel(const int32_t *__restrict__ task_token, const int32_t *__restrict__ task_expert,
                   const float *__restrict__ task_gate, int64_t M, int64_t N, int L,
                   const int32_t *__restrict__ cnt, int cap, float *__restrict__ Gm,
                   int32_t *__restrict__ c_tok, int32_t *__restrict__ c_exp,
                   float *__restrict__ c_gate, int32_t *__restrict__ c_count,
                   const int32_t *__restrict__ covered, int *status) {
    grid_dependency_wait();
    grid_dependents_launch();
    const unsigned lane = lane_id();
    if (blockIdx.x == 0 && threadIdx.x == 0 && (int64_t)*covered != M)
        set_status(status, OMNI_DEV_BAD_SCHEDULE);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t chunk = 32 * kSplitRounds;
    for (int64_t c0 = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * chunk;
         c0 < M; c0 += nwarps * chunk) {
        unsigned my_mask = 0;                         // lane r: the CUDA-core tasks of round r
#pragma unroll 4
        for (int r = 0; r < kSplitRounds; ++r) {
            const int64_t m = c0 + r * 32 + lane;
            bool cold = false;
            if (m < M) {
                int32_t t = task_token[m], e = task_expert[m];
                if (t < 0 || t >= L || e < 0 || (int64_t)e >= N) {
                    set_status(status, OMNI_DEV_BAD_SCHEDULE);
                    t = t < 0 || t >= L ? 0 : t;
                    e = e < 0 || (int64_t)e >= N ? 0 : e;
                }
                const int32_t v = cnt[e];
                if (v < 0)
                    Gm[(size_t)t * cap + (-v - 1)] = task_gate[m];
                else
                    cold = true;
            }
            const unsigned bal = __ballot_sync(0xffffffffu, cold);
            if (lane == (unsigned)r) my_mask = bal;
        }
        const int mine = __popc(my_mask);
        const int incl = warp_iscan(mine);
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        if (total == 0) continue;
        int base = 0;
        if (lane == 0) base = atomicAdd(c_count, total);
        base = __shfl_sync(0xffffffffu, base, 0) + incl - mine;   // this lane's round starts here
        for (int r = 0; r < kSplitRounds; ++r) {
            const unsigned bal = __shfl_sync(0xffffffffu, my_mask, r);
            const int at0 = __shfl_sync(0xffffffffu, base, r);
            if (bal == 0) continue;
            if ((bal >> lane) & 1u) {
                const int64_t m = c0 + r * 32 + lane;
                int32_t t = task_token[m], e = task_expert[m];
                t = t < 0 || t >= L ? 0 : t;
                e = e < 0 || (int64_t)e >= N ? 0 : e;
                const int at = at0 + __popc(bal & lanemask_lt());
                c_tok[at] = t;
                c_exp[at] = e;
                c_gate[at] = task_gate[m];
            }
        }
    }
}

// ------------------------------------------------------ 7-8. tile GEMMs
// Persistent, warp-specialised: warp 0 issues TMA loads into a 4-stage ring
// (A: 128 rows x 64 K, B: two boxes of 128 rows x 64 K), warp 1 issues
// tcgen05.mma kind::f16 into one of two 256-column TMEM accumulators, warps
// 2-9 drain the other one (warp w reads TMEM lanes 32 (w % 4) .. + 31 and
// half of the columns).
//   kEpiGate: A = x [L, d], B = W_D [cap, d]; n tiles over the E_pad dense
//             columns; the epilogue writes P = bf16(G . SiLU(H)).
//   kEpiAdd:  A = P [L, cap], B = V_D^T [d, cap]; K runs over the E_pad dense
//             columns; the epilogue adds the fp32 tile into y.
constexpr int BM = 128, BN = 256, BK = kSwK, STAGES = 4;
constexpr int kBoxRows = BN / 2;
constexpr int kTileBytesA = BM * BK * 2;         // 16 KB
constexpr int kBoxBytesB = kBoxRows * BK * 2;    // 16 KB
constexpr int kTileBytesB = 2 * kBoxBytesB;      // 32 KB
constexpr uint32_t kTmemCols = 2 * BN;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr uint32_t kIdesc = umma_idesc_bf16(BM, BN);

enum : int { kEpiGate = 0, kEpiAdd = 1 };

struct __align__(1024) GemmSmem {
    uint8_t a[STAGES][kTileBytesA];
    uint8_t b[STAGES][kTileBytesB];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint32_t tmem_base;
    int abort;
};

struct DenseGemm {
    int M;                  // tokens
    int d;
    int cap;                // row stride of G and P, columns of V_D^T
    const int32_t *ehot;    // number of dense experts (capped at cap here)
    const float *G;         // kEpiGate
    uint16_t *P;            // kEpiGate output
    float *y;               // kEpiAdd
    int *status;
};

__device__ __forceinline__ float silu_f32(float z) { return z / (1.f + __expf(-z)); }

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
dense_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                  const DenseGemm p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    GemmSmem &sm = *reinterpret_cast<GemmSmem *>(smem_raw + pad);
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
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
    grid_dependency_wait();
    grid_dependents_launch();
    // extents: the number of dense experts was written by earlier kernels
    const int E = dense_count(p.ehot, p.cap);
    const int Ep = (E + 255) & ~255;
    const int nk = EPI == kEpiGate ? p.d / BK : Ep / BK;
    const int ntn = EPI == kEpiGate ? Ep / BN : (Ep > 0 ? p.d / BN : 0);
    const int ntiles = ((p.M + BM - 1) / BM) * ntn;

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer
            int it = 0, issued_from = 0;
            for (int tile = blockIdx.x; tile < ntiles && !sm.abort; tile += gridDim.x) {
                const int m0 = (tile / ntn) * BM;
                const int r0 = (tile % ntn) * BN;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (it >= STAGES &&
                        !mbar_wait(&sm.empty[s], (uint32_t)(((it / STAGES) - 1) & 1), status)) {
                        sm.abort = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.full[s], kTileBytesA + kTileBytesB);
                    tma_load_2d(sm.a[s], &tm_a, kb * BK, m0, &sm.full[s]);
                    tma_load_2d(sm.b[s], &tm_b, kb * BK, r0, &sm.full[s]);
                    tma_load_2d(sm.b[s] + kBoxBytesB, &tm_b, kb * BK, r0 + kBoxRows, &sm.full[s]);
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
                    for (int k = 0; k < BK / 16; ++k)
                        umma_bf16(acc, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), kIdesc,
                                  (kb > 0 || k > 0) ? 1u : 0u);
                    umma_commit(&sm.empty[s]);
                }
                umma_commit(&sm.tfull[buf]);
            }
            if (!ok) sm.abort = 1;
        }
        __syncwarp();
    } else {
        // ---- epilogue
        const int quarter = warp & 3;
        const int half = (warp - 2) >> 2;
        int lt = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++lt) {
            const int buf = lt & 1;
            if (!mbar_wait(&sm.tfull[buf], (uint32_t)((lt >> 1) & 1), status)) break;
            tc_fence_after();
            const int m0 = (tile / ntn) * BM;
            const int tn = tile % ntn;
            const int row = m0 + quarter * 32 + (int)lane;
            const uint32_t tb = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
#pragma unroll
            for (int c = 0; c < kBoxRows / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tb + (uint32_t)(half * kBoxRows + 32 * c), r);
                const int col = tn * BN + half * kBoxRows + 32 * c;
                if (row >= p.M) continue;
                if (EPI == kEpiGate) {
                    // P = G . SiLU(H) for 32 dense columns of this token
                    const float4 *gr = reinterpret_cast<const float4 *>(p.G + (size_t)row * p.cap + col);
                    uint32_t hp[16];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 g = gr[q];
                        const float a0 = g.x * silu_f32(__uint_as_float(r[4 * q]));
                        const float a1 = g.y * silu_f32(__uint_as_float(r[4 * q + 1]));
                        const float a2 = g.z * silu_f32(__uint_as_float(r[4 * q + 2]));
                        const float a3 = g.w * silu_f32(__uint_as_float(r[4 * q + 3]));
                        const __nv_bfloat162 lo = __floats2bfloat162_rn(a0, a1);
                        const __nv_bfloat162 hi = __floats2bfloat162_rn(a2, a3);
                        hp[2 * q] = *reinterpret_cast<const uint32_t *>(&lo);
                        hp[2 * q + 1] = *reinterpret_cast<const uint32_t *>(&hi);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(p.P + (size_t)row * p.cap + col);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(hp[4 * q], hp[4 * q + 1], hp[4 * q + 2], hp[4 * q + 3]);
                } else {
                    float4 *dst = reinterpret_cast<float4 *>(p.y + (size_t)row * p.d + col);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 prev = dst[q];
                        dst[q] = make_float4(prev.x + __uint_as_float(r[4 * q]),
                                             prev.y + __uint_as_float(r[4 * q + 1]),
                                             prev.z + __uint_as_float(r[4 * q + 2]),
                                             prev.w + __uint_as_float(r[4 * q + 3]));
                    }
                }
            }
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
cudaError_t launch_dense_gemm(const CUtensorMap &a, const CUtensorMap &b, const DenseGemm &p,
                              int max_tiles, cudaStream_t st) {
    const int smem = (int)sizeof(GemmSmem) + 1024;
    const cudaError_t e = cudaFuncSetAttribute(dense_gemm_kernel<EPI>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int sms = device_sm_count();
    int grid = max_tiles < sms ? max_tiles : sms;
    if (grid < 1) grid = 1;
    return launch(dense_gemm_kernel<EPI>, dim3(grid), dim3(kThreads), (size_t)smem, st, a, b, p);
}

}  // namespace

// ------------------------------------------------------------------- host
DenseWs dense_ws_of(const Sizes &sz, void *ws, const WsLayout &lay) {
    DenseWs o;
    o.cnt = ws_at<int32_t>(ws, lay.dz_cnt);
    o.ghot = ws_at<int32_t>(ws, lay.dz_ghot);
    o.ehot = ws_at<int32_t>(ws, lay.d_ehot);
    o.ccount = ws_at<int32_t>(ws, lay.dz_ccount);
    o.list = ws_at<int32_t>(ws, lay.d_list);
    o.whot = ws_at<uint16_t>(ws, lay.d_whot);
    o.vt = ws_at<uint16_t>(ws, lay.d_vt);
    o.G = ws_at<float>(ws, lay.d_G);
    o.P = ws_at<uint16_t>(ws, lay.d_P);
    o.c_tok = ws_at<int32_t>(ws, lay.d_ctok);
    o.c_exp = ws_at<int32_t>(ws, lay.d_cexp);
    o.c_gate = ws_at<float>(ws, lay.d_cgate);
    o.cap = sz.dense_cap;
    o.thr = sz.dense_thr;
    return o;
}

cudaError_t launch_dense_prepare(const uint16_t *W, const uint16_t *V, const Sizes &sz,
                                 const int32_t *task_token, const int32_t *task_expert,
                                 const float *task_gate, const int32_t *group_offsets,
                                 const int32_t *active_groups, const int32_t *num_active,
                                 const DenseWs &o, int *status, cudaStream_t st) {
    const int sms = device_sm_count();
    const int64_t G = sz.G;
    auto grid_for = [&](int64_t warps_needed) {
        int64_t g = (warps_needed + 7) / 8;               // 8 warps per CTA
        if (g > (int64_t)sms * 8) g = (int64_t)sms * 8;
        return (unsigned)(g < 1 ? 1 : g);
    };
    cudaError_t e = launch(dense_use_kernel, dim3(grid_for((sz.M + 31) / 32)), dim3(256), 0, st,
                           task_expert, sz.M, group_offsets, sz.B, sz.N, o.cnt, status);
    if (e != cudaSuccess) return e;
    e = launch(dense_mark_kernel, dim3(grid_for(G)), dim3(256), 0, st, (const int32_t *)o.cnt,
               group_offsets, active_groups, num_active, G, sz.B, sz.N, sz.M, o.thr, o.ghot,
               o.ccount + 1, status);
    if (e != cudaSuccess) return e;
    // ghot has G + 1 entries (the last one zero): its scan gives hoff[G] = E
    if ((e = launch_exclusive_scan(o.ghot, G + 1, o.ehot, st)) != cudaSuccess) return e;
    e = launch(dense_list_kernel, dim3(grid_for(G)), dim3(256), 0, st, (const int32_t *)o.ghot,
               active_groups, num_active, G, sz.B, sz.N, o.thr, o.cap, o.cnt, o.list);
    if (e != cudaSuccess) return e;
    e = launch(dense_gather_kernel, dim3((unsigned)(sms * 4)), dim3(kGatherThreads), 0, st, W, V,
               sz.d, sz.L, sz.N, (const int32_t *)o.list, (const int32_t *)o.ehot, o.cap, o.whot,
               o.vt, o.G);
    if (e != cudaSuccess) return e;
    const int64_t chunks = (sz.M + 32 * kSplitRounds - 1) / (32 * kSplitRounds);
    return launch(dense_split_kernel, dim3(grid_for(chunks)), dim3(256), 0, st, task_token,
                  task_expert, task_gate, sz.M, sz.N, sz.L, (const int32_t *)o.cnt, o.cap, o.G,
                  o.c_tok, o.c_exp, o.c_gate, o.ccount, (const int32_t *)(o.ccount + 1), status);
}

cudaError_t launch_dense_gemms(const uint16_t *x, const Sizes &sz, const DenseWs &o, float *y,
                               int *status, cudaStream_t st) {
    CUtensorMap tm_x, tm_w, tm_p, tm_v;
    if (!make_sw128_map(&tm_x, x, sz.L, sz.d, BM) ||
        !make_sw128_map(&tm_w, o.whot, o.cap, sz.d, kBoxRows) ||
        !make_sw128_map(&tm_p, o.P, sz.L, o.cap, BM) ||
        !make_sw128_map(&tm_v, o.vt, sz.d, o.cap, kBoxRows))
        return cudaErrorInvalidValue;
    DenseGemm p;
    p.M = sz.L;
    p.d = sz.d;
    p.cap = o.cap;
    p.ehot = o.ehot;
    p.G = o.G;
    p.P = o.P;
    p.y = y;
    p.status = status;
    const int mt = (sz.L + BM - 1) / BM;
    cudaError_t e = launch_dense_gemm<kEpiGate>(tm_x, tm_w, p, mt * (o.cap / BN), st);
    if (e != cudaSuccess) return e;
    return launch_dense_gemm<kEpiAdd>(tm_p, tm_v, p, mt * (sz.d / BN), st);
}

}  // namespace omni

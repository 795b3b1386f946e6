// expert.cu -- grouped expert stage on sm_100a.
//
// "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale"
// (rainbus review page, method paragraph, steps 1 and 3; gist.science
// summary, section 2.2 "Grouped GEMM"): for each active group q,
//     O_q = (G_q . SiLU(X_q W_q^T)) V_q,   y[t] += O_q[t],
// where W_q, V_q are the rows of the group's active experts, X_q the rows of
// its tokens and G_q the gate of each (token, expert) task, 0 elsewhere.
// sigma is read as SiLU (each atomic expert has a single w_in).
//
// Two kernels, no atomics on y:
//   1. group pass (expert-centric, per group as the pages have it):
//      P_q = G_q . SiLU(X_q W_q^T) for the task pairs only (G_q is about 8%
//      dense for 4096 tokens over 1.7M experts).  Every warp owns a
//      contiguous share of the sorted tasks and cuts it where the group
//      changes; it orders its tasks by expert id (a counting sort inside
//      each group) and goes expert by expert, loading each W row once
//      (cp.async, 16 bytes per lane, into the warp's own shared-memory ring)
//      and using it for every token of the group that chose it.  The x rows
//      of the tasks stream through a second ring, kStages-1 tasks ahead.  Each task's p = g * SiLU(x_t . w_e) is
//      written with its expert id into a slot of its token.
//   2. token pass: y[t] = sum over the token's slots of p * V[e], one warp
//      per token, V rows prefetched the same way; y is written once per
//      token.  This is O_q = P_q V_q plus the scatter-add, regrouped by
//      token: on B200 the fp32 reductions of per-group partial rows into y
//      (16-byte red.global.add.v4.f32, one L2 sector operation each) ran at
//      about 3 TB/s and cost more than the HBM gather they were meant to
//      follow, while V rows are used about 1.1 times per group at this scale.
// A warp that shares a group with its neighbour reloads the experts common
// to both halves (about one row per warp boundary).  No kernel here waits on
// another warp or CTA.
#include "omni_common.cuh"
#include "omni_internal.h"

namespace omni {
namespace {

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &u, float *f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// ---------------------------------------------------------- common parts
constexpr int kSub = 256;                 // tasks staged per sub-range

// Per-warp scratch of the group pass for one sub-range of tasks.
struct WarpScratch {
    int tok[kSub];
    int exp[kSub];
    float gate[kSub];
    uint16_t rank[kSub];          // rank of the task's expert in the sub-range's expert list
    uint16_t order[kSub];         // segment tasks, expert-major
    int slot[kSub];               // the task's slot among its token's K slots
    int start[kSub + 4];          // per expert rank: first position in order[] (+ padding)
    int elist[kSub];              // distinct experts of the sub-range, ascending
    uint32_t bitmap[OMNI_MAX_B / 32];
    int word_prefix[OMNI_MAX_B / 32];
};
static_assert(sizeof(WarpScratch) % 16 == 0, "scratch keeps 16-byte alignment");

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                 ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// copy one bf16 row of 256*VPL elements into shared memory, 16 bytes per lane
template <int VPL>
__device__ __forceinline__ void row_async(uint8_t *dst, const uint16_t *src, unsigned lane) {
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int v = 0; v < VPL; ++v) cp_async16(dst + (size_t)(v * 32 + lane) * 16, s4 + v * 32 + lane);
}

template <int VPL, int STAGES, int EXTRA>
struct WarpSmem {
    static constexpr int kRowBytes = 512 * VPL;
    static constexpr int kWarpBytes = STAGES * kRowBytes + EXTRA;
    static constexpr int kFit = (227 * 1024) / kWarpBytes;
    static constexpr int kWarps = kFit > 16 ? 16 : kFit;
    static_assert(kWarps >= 2, "too little shared memory per warp");
    static_assert(kWarpBytes % 16 == 0, "per-warp areas stay 16-byte aligned");
};

template <int VPL>
struct GateCfg {
    // tasks in flight per warp; each stage holds a W row and an x row
    static constexpr int kStages = VPL <= 1 ? 10 : (VPL <= 2 ? 8 : (VPL <= 4 ? 6 : 4));
    using Smem = WarpSmem<VPL, 2 * kStages, (int)sizeof(WarpScratch)>;
};
template <int VPL>
struct CombineCfg {
    static constexpr int kStages = VPL <= 2 ? 10 : (VPL <= 4 ? 8 : 5);
    static constexpr int kWarps = 4;                      // per CTA; several CTAs per SM
    static constexpr int kRowBytes = 512 * VPL;
    static constexpr int kSmem = kWarps * kStages * kRowBytes;
};

// ------------------------------------------------------- 1. group pass
template <int VPL>
__global__ void __launch_bounds__(32 * GateCfg<VPL>::Smem::kWarps, 1)
group_gate_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ W, int L, int N,
                  int B, int K, int M, int per_warp, const int32_t *__restrict__ task_token,
                  const int32_t *__restrict__ task_expert, const float *__restrict__ task_gate,
                  int *__restrict__ tok_count, int2 *__restrict__ tok_slots, int *status) {
    using Cfg = GateCfg<VPL>;
    using Sm = typename Cfg::Smem;
    constexpr int D = 256 * VPL;
    constexpr int S = Cfg::kStages;
    constexpr int RB = Sm::kRowBytes;
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    uint8_t *ring = smem + (size_t)warp * Sm::kWarpBytes;          // S W rows, then S x rows
    WarpScratch &sc = *reinterpret_cast<WarpScratch *>(ring + 2 * S * RB);
    static_assert(Sm::kWarpBytes == 2 * S * RB + (int)sizeof(WarpScratch), "per-warp layout");
    const int nwords = (B + 31) >> 5;

    const int64_t gw = (int64_t)blockIdx.x * Sm::kWarps + warp;
    const int64_t a0 = gw * per_warp;
    const int64_t a1 = a0 + per_warp < M ? a0 + per_warp : M;

    for (int64_t sub = a0; sub < a1; sub += kSub) {
        const int n = (int)(a1 - sub < kSub ? a1 - sub : kSub);
        __syncwarp();
        for (int j = lane; j < n; j += 32) {
            int t = task_token[sub + j], e = task_expert[sub + j];
            if (e < 0 || e >= N || t < 0 || t >= L) {
                set_status(status, OMNI_DEV_BAD_SCHEDULE);
                e = e < 0 || e >= N ? 0 : e;
                t = t < 0 || t >= L ? 0 : t;
            }
            sc.tok[j] = t;
            sc.exp[j] = e;
            sc.gate[j] = task_gate[sub + j];
            // claim the task's slot now, 32 tasks per round trip
            sc.slot[j] = atomicAdd(&tok_count[t], 1);
        }
        __syncwarp();
        // ---- setup for the whole sub-range: tasks sorted by expert id (the
        // sub-range is in (group, token, expert) order, so this is a per-group
        // counting sort on e - q*B), expert list, expert-major task order
        for (int k = lane; k <= n; k += 32) sc.start[k] = 0;
        __syncwarp();
        int n_e = 0;
        for (int js = 0; js < n;) {
            const int q = sc.exp[js] / B;
            int je = n;
            for (int j0 = js + 1; j0 < n; j0 += 32) {
                const int j = j0 + (int)lane;
                const bool brk = j < n && sc.exp[j] / B != q;
                const unsigned bal = __ballot_sync(0xffffffffu, brk);
                if (bal) {
                    je = j0 + __ffs(bal) - 1;
                    break;
                }
            }
            const int64_t ebase = (int64_t)q * B;
            for (int w = lane; w < nwords; w += 32) sc.bitmap[w] = 0u;
            __syncwarp();
            for (int j = js + lane; j < je; j += 32) {
                const int r = (int)(sc.exp[j] - ebase);
                atomicOr(&sc.bitmap[r >> 5], 1u << (r & 31));
            }
            __syncwarp();
            const uint32_t wbits = lane < (unsigned)nwords ? sc.bitmap[lane] : 0u;
            const int cnt = __popc(wbits);
            const int incl = warp_iscan(cnt);
            if (lane < (unsigned)nwords) {
                sc.word_prefix[lane] = incl - cnt;
                uint32_t bits = wbits;
                int pos = n_e + incl - cnt;
                while (bits) {
                    const int b = __ffs(bits) - 1;
                    sc.elist[pos++] = (int)(ebase + lane * 32 + b);
                    bits &= bits - 1;
                }
            }
            __syncwarp();
            // per task: global expert rank; per expert: task count (task order)
            for (int j0 = js; j0 < je; j0 += 32) {
                const int j = j0 + (int)lane;
                const bool in = j < je;
                int rk = 0x7fffffff;
                if (in) {
                    const int r = (int)(sc.exp[j] - ebase);
                    const int wd = r >> 5;
                    rk = n_e + sc.word_prefix[wd] + __popc(sc.bitmap[wd] & ((1u << (r & 31)) - 1u));
                    sc.rank[j] = (uint16_t)rk;
                }
                const unsigned peers = __match_any_sync(0xffffffffu, rk);
                if (in && (peers & lanemask_lt()) == 0) sc.start[rk + 1] += __popc(peers);
                __syncwarp();
            }
            n_e += __shfl_sync(0xffffffffu, incl, 31);
            js = je;
        }
        // exclusive scan of the counts -> start[k]
        {
            int carry = 0;
            for (int k0 = 0; k0 <= n_e; k0 += 32) {
                const int k = k0 + (int)lane;
                const int v = k <= n_e ? sc.start[k] : 0;
                const int inc = warp_iscan(v);
                if (k <= n_e) sc.start[k] = carry + inc;
                carry += __shfl_sync(0xffffffffu, inc, 31);
            }
        }
        __syncwarp();
        // place tasks expert-major, keeping task order inside an expert
        for (int j0 = 0; j0 < n; j0 += 32) {
            const int j = j0 + (int)lane;
            const bool in = j < n;
            const int rk = in ? (int)sc.rank[j] : 0x7fffffff;
            const unsigned peers = __match_any_sync(0xffffffffu, rk);
            int base = 0;
            if (in) base = sc.start[rk];
            if (in) sc.order[base + __popc(peers & lanemask_lt())] = (uint16_t)j;
            __syncwarp();
            if (in && (peers & lanemask_lt()) == 0) sc.start[rk] += __popc(peers);
            __syncwarp();
        }
        // ---- expert-major pass over the sub-range: p for every task.
        // Stream unit = one task: its x row (x ring slot i % S) and, for the
        // first task of an expert, the expert's W row (W ring slot k % S).
        // Tasks i .. i+S-1 span at most S experts, so a W slot is refilled only
        // after every task of its previous expert has been computed.
        uint8_t *wring = ring;
        uint8_t *xring = ring + S * RB;
        auto issue = [&](int i) {
            const int j = sc.order[i];
            const int k = sc.rank[j];
            if (i == 0 || sc.rank[sc.order[i - 1]] != k)
                row_async<VPL>(wring + (k % S) * RB, W + (size_t)sc.elist[k] * D, lane);
            row_async<VPL>(xring + (i % S) * RB, x + (size_t)sc.tok[j] * D, lane);
        };
#pragma unroll 1
        for (int i = 0; i < S - 1; ++i) {
            if (i < n) issue(i);
            cp_async_commit();
        }
        for (int i = 0; i < n; ++i) {
            cp_async_wait<S - 2>();                // task i's rows have landed
            __syncwarp();
            if (i + S - 1 < n) issue(i + S - 1);
            cp_async_commit();
            const int j = sc.order[i];
            const int k = sc.rank[j];
            const uint4 *wr = reinterpret_cast<const uint4 *>(wring + (k % S) * RB);
            const uint4 *xr = reinterpret_cast<const uint4 *>(xring + (i % S) * RB);
            float h = 0.f;
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                float xf[8], wf[8];
                bf16x8_to_f32(xr[v * 32 + lane], xf);
                bf16x8_to_f32(wr[v * 32 + lane], wf);
#pragma unroll
                for (int c = 0; c < 8; ++c) h = fmaf(xf[c], wf[c], h);
            }
            h = warp_sum(h);
            if (lane == 0) {
                const float p = sc.gate[j] * (h / (1.f + __expf(-h)));
                const int slot = sc.slot[j];
                if (slot < K)
                    tok_slots[(size_t)sc.tok[j] * K + slot] = make_int2(sc.exp[j], __float_as_int(p));
                else
                    set_status(status, OMNI_DEV_BAD_SCHEDULE);
            }
        }
        // drain the remaining copies before the ring is reused
        cp_async_wait<0>();
        __syncwarp();
    }
}

// ------------------------------------------------------- 2. token pass
// One warp per token (grid-stride): y[t] (+)= sum_s p_s * V[e_s].
template <int VPL>
__global__ void __launch_bounds__(32 * CombineCfg<VPL>::kWarps)
token_combine_kernel(const uint16_t *__restrict__ V, int L, int N, int K,
                     const int *__restrict__ tok_count, const int2 *__restrict__ tok_slots,
                     float *__restrict__ y, int accumulate, int *status) {
    using Cfg = CombineCfg<VPL>;
    constexpr int D = 256 * VPL;
    constexpr int S = Cfg::kStages;
    constexpr int RB = Cfg::kRowBytes;
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    uint8_t *ring = smem + (size_t)warp * S * RB;
    const int nwarps = gridDim.x * Cfg::kWarps;
    for (int t = blockIdx.x * Cfg::kWarps + warp; t < L; t += nwarps) {
        int n = tok_count[t];
        if (n > K) {
            set_status(status, OMNI_DEV_BAD_SCHEDULE);
            n = K;
        }
        const int2 *sl = tok_slots + (size_t)t * K;
        // expert ids of the token's first 32 slots, one per lane
        int2 mine = lane < (unsigned)n ? sl[lane] : make_int2(0, 0);
        if (mine.x < 0 || mine.x >= N) mine.x = 0;
        auto expert_of = [&](int s) -> int {
            // slot s lives in lane s % 32 of the block of 32 slots holding it
            return __shfl_sync(0xffffffffu, mine.x, s & 31);
        };
        float acc[VPL * 8];
#pragma unroll
        for (int c = 0; c < VPL * 8; ++c) acc[c] = 0.f;
#pragma unroll
        for (int s = 0; s < S - 1; ++s) {
            if (s < n) row_async<VPL>(ring + (s % S) * RB, V + (size_t)expert_of(s) * D, lane);
            cp_async_commit();
        }
        for (int s = 0; s < n; ++s) {
            cp_async_wait<S - 2>();
            __syncwarp();
            const float p = __int_as_float(__shfl_sync(0xffffffffu, mine.y, s & 31));
            const int sn = s + S - 1;
            int en = 0;
            if (sn < n) {
                if ((sn >> 5) == (s >> 5)) {
                    en = expert_of(sn);                // held by the lanes of this block
                } else {
                    const int2 nx = sl[sn];            // next block: same address in every lane
                    en = (nx.x < 0 || nx.x >= N) ? 0 : nx.x;
                }
                row_async<VPL>(ring + (sn % S) * RB, V + (size_t)en * D, lane);
            }
            cp_async_commit();
            const uint4 *vr = reinterpret_cast<const uint4 *>(ring + (s % S) * RB);
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                float vf[8];
                bf16x8_to_f32(vr[v * 32 + lane], vf);
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[8 * v + c] = fmaf(p, vf[c], acc[8 * v + c]);
            }
            if (((s + 1) & 31) == 0 && s + 1 < n) {
                // next block of 32 slots
                mine = (s + 1 + (int)lane) < n ? sl[s + 1 + lane] : make_int2(0, 0);
                if (mine.x < 0 || mine.x >= N) mine.x = 0;
            }
        }
        cp_async_wait<0>();
        __syncwarp();
        float *yr = y + (size_t)t * D;
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            float4 *dst = reinterpret_cast<float4 *>(yr + (size_t)(v * 32 + lane) * 8);
            float4 a = make_float4(acc[8 * v], acc[8 * v + 1], acc[8 * v + 2], acc[8 * v + 3]);
            float4 b = make_float4(acc[8 * v + 4], acc[8 * v + 5], acc[8 * v + 6], acc[8 * v + 7]);
            if (accumulate) {
                const float4 oa = dst[0], ob = dst[1];
                a.x += oa.x; a.y += oa.y; a.z += oa.z; a.w += oa.w;
                b.x += ob.x; b.y += ob.y; b.z += ob.z; b.w += ob.w;
            }
            dst[0] = a;
            dst[1] = b;
        }
    }
}

template <int VPL>
cudaError_t launch_vpl(const uint16_t *x, const uint16_t *W, const uint16_t *V, const Sizes &sz,
                       const int32_t *tt, const int32_t *te, const float *tg, float *y,
                       bool accumulate, int *tok_count, int2 *tok_slots, int *status,
                       cudaStream_t st) {
    using G = GateCfg<VPL>;
    using C = CombineCfg<VPL>;
    constexpr int gwarps = G::Smem::kWarps;
    constexpr int gsmem = gwarps * G::Smem::kWarpBytes;
    cudaError_t e = cudaFuncSetAttribute(group_gate_kernel<VPL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, gsmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(token_combine_kernel<VPL>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    const int sms = device_sm_count();
    if ((e = cudaMemsetAsync(tok_count, 0, sizeof(int) * (size_t)sz.L, st)) != cudaSuccess) return e;
    {
        const int64_t warps = (int64_t)sms * gwarps;
        int64_t per_warp = (sz.M + warps - 1) / warps;
        if (per_warp < 32) per_warp = 32;
        const int64_t needed = (sz.M + per_warp - 1) / per_warp;      // warps with work
        const int grid = (int)((needed + gwarps - 1) / gwarps);
        group_gate_kernel<VPL><<<grid, 32 * gwarps, gsmem, st>>>(
            x, W, sz.L, (int)sz.N, sz.B, sz.K, (int)sz.M, (int)per_warp, tt, te, tg, tok_count,
            tok_slots, status);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        int per_sm = (227 * 1024) / C::kSmem;
        if (per_sm < 1) per_sm = 1;
        if (per_sm > 8) per_sm = 8;
        int64_t grid = (int64_t)sms * per_sm;
        const int64_t need = (sz.L + C::kWarps - 1) / C::kWarps;
        if (grid > need) grid = need;
        token_combine_kernel<VPL><<<(unsigned)grid, 32 * C::kWarps, C::kSmem, st>>>(
            V, sz.L, (int)sz.N, sz.K, tok_count, tok_slots, y, accumulate ? 1 : 0, status);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_grouped_expert(const uint16_t *x, const uint16_t *W, const uint16_t *V,
                                  const Sizes &sz, const int32_t *task_token,
                                  const int32_t *task_expert, const float *task_gate,
                                  float *y, bool accumulate, void *ws, const WsLayout &lay,
                                  cudaStream_t st) {
    int *status = ws_at<int>(ws, lay.hdr);
    int *tok_count = ws_at<int>(ws, lay.tok_count);
    int2 *tok_slots = ws_at<int2>(ws, lay.tok_slots);
    switch (sz.d / 256) {
#define OMNI_CASE(n) \
        case n: return launch_vpl<n>(x, W, V, sz, task_token, task_expert, task_gate, y, accumulate, \
                                     tok_count, tok_slots, status, st);
        OMNI_CASE(1) OMNI_CASE(2) OMNI_CASE(3) OMNI_CASE(4)
        OMNI_CASE(5) OMNI_CASE(6) OMNI_CASE(7) OMNI_CASE(8)
#undef OMNI_CASE
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace omni

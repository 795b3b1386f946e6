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
// Design.  The cost is the gather of the active expert rows (2*d bytes each
// for W and V) from HBM; G_q is sparse (about 8% dense for 4096 tokens over
// 1.7M experts), so only the task pairs are computed, on CUDA cores, and the
// kernel is built to keep many independent row loads in flight:
//   - every warp owns a contiguous share of the sorted task array (no work
//     list, no claiming); it cuts its share where the group changes;
//   - inside a group segment the warp goes expert by expert (expert-major):
//     the W and V rows of an expert are loaded once and used for every token
//     of the segment that chose it.  Rows are prefetched kStages-1 experts
//     ahead with cp.async (16 bytes per lane) into the warp's own shared-
//     memory ring, so each warp keeps several rows in flight without
//     spending registers on them;
//   - per task the warp computes h = x_t . w_e (warp reduction),
//     p = g * SiLU(h) and adds p * v_e into y[t] with vector reductions
//     (red.global.add.v4.f32); y is L2-resident for typical L.  The x row of
//     the next task is loaded while the current one is computed.
// A warp that shares a group with its neighbour reloads the experts common
// to both halves (about one row per warp boundary).  No waits on other warps
// or other CTAs exist in this kernel.
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

// ---------------------------------------------------------- main kernel
constexpr int kSub = 256;                 // tasks staged per sub-range

// Per-warp scratch for one sub-range of tasks.
struct WarpScratch {
    int tok[kSub];
    int exp[kSub];
    float gate[kSub];
    uint16_t rank[kSub];          // rank of the task's expert within its segment
    uint16_t order[kSub];         // segment tasks, expert-major
    int start[kSub + 4];          // per expert rank: first position in order[] (+ padding)
    uint16_t rlist[kSub];         // distinct experts of the segment (r = e - q*B)
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

template <int VPL>
struct ExpertCfg {
    static constexpr int kD = 256 * VPL;                 // d
    static constexpr int kRowBytes = 2 * kD;             // one bf16 row
    static constexpr int kPairBytes = 2 * kRowBytes;     // W row + V row
    static constexpr int kStages = VPL <= 1 ? 6 : (VPL <= 2 ? 5 : (VPL <= 4 ? 4 : 3));
    static constexpr int kWarpBytes = kStages * kPairBytes + (int)sizeof(WarpScratch);
    static constexpr int kWarpsFit = (227 * 1024) / kWarpBytes;
    static constexpr int kWarps = kWarpsFit > 16 ? 16 : kWarpsFit;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kSmem = kWarps * kWarpBytes;
    static_assert(kWarps >= 2, "too little shared memory per warp");
    static_assert(kPairBytes % 16 == 0, "ring slots stay 16-byte aligned");
};

template <int VPL>
__global__ void __launch_bounds__(ExpertCfg<VPL>::kThreads, 1)
grouped_expert_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ W,
                      const uint16_t *__restrict__ V, int L, int N, int B, int M, int per_warp,
                      const int32_t *__restrict__ task_token,
                      const int32_t *__restrict__ task_expert,
                      const float *__restrict__ task_gate, float *__restrict__ y, int *status) {
    using Cfg = ExpertCfg<VPL>;
    constexpr int D = Cfg::kD;
    constexpr int S = Cfg::kStages;
    constexpr int RB = Cfg::kRowBytes;
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    uint8_t *ring = smem + (size_t)warp * Cfg::kWarpBytes;
    WarpScratch &sc = *reinterpret_cast<WarpScratch *>(ring + S * Cfg::kPairBytes);
    const int nwords = (B + 31) >> 5;

    const int64_t gw = (int64_t)blockIdx.x * Cfg::kWarps + warp;
    const int64_t a0 = gw * per_warp;
    const int64_t a1 = a0 + per_warp < M ? a0 + per_warp : M;

    // issue the cp.async copies of one expert's W and V rows into ring slot k % S
    auto issue = [&](int k, int64_t e) {
        uint8_t *slot = ring + (k % S) * Cfg::kPairBytes;
        const uint4 *wsrc = reinterpret_cast<const uint4 *>(W + e * D);
        const uint4 *vsrc = reinterpret_cast<const uint4 *>(V + e * D);
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            cp_async16(slot + (size_t)(v * 32 + lane) * 16, wsrc + v * 32 + lane);
            cp_async16(slot + RB + (size_t)(v * 32 + lane) * 16, vsrc + v * 32 + lane);
        }
    };

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
        }
        __syncwarp();
        int js = 0;
        while (js < n) {
            // ---- segment [js, je): the run of tasks of one group
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
            // distinct experts, ranked by expert id
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
            const int n_e = __shfl_sync(0xffffffffu, incl, 31);
            if (lane < (unsigned)nwords) {
                sc.word_prefix[lane] = incl - cnt;
                uint32_t bits = wbits;
                int pos = incl - cnt;
                while (bits) {
                    const int b = __ffs(bits) - 1;
                    sc.rlist[pos++] = (uint16_t)(lane * 32 + b);
                    bits &= bits - 1;
                }
            }
            for (int k = lane; k <= n_e; k += 32) sc.start[k] = 0;
            __syncwarp();
            // start the first S-1 experts' rows while the ordering is built
#pragma unroll
            for (int k = 0; k < S - 1; ++k) {
                if (k < n_e) issue(k, ebase + sc.rlist[k]);
                cp_async_commit();
            }
            // per task: expert rank; per expert: task count (deterministic,
            // in task order)
            for (int j0 = js; j0 < je; j0 += 32) {
                const int j = j0 + (int)lane;
                const bool in = j < je;
                int rk = 0x7fffffff;
                if (in) {
                    const int r = (int)(sc.exp[j] - ebase);
                    const int wd = r >> 5;
                    rk = sc.word_prefix[wd] + __popc(sc.bitmap[wd] & ((1u << (r & 31)) - 1u));
                    sc.rank[j] = (uint16_t)rk;
                }
                const unsigned peers = __match_any_sync(0xffffffffu, rk);
                if (in && (peers & lanemask_lt()) == 0) sc.start[rk + 1] += __popc(peers);
                __syncwarp();
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
            for (int j0 = js; j0 < je; j0 += 32) {
                const int j = j0 + (int)lane;
                const bool in = j < je;
                const int rk = in ? (int)sc.rank[j] : 0x7fffffff;
                const unsigned peers = __match_any_sync(0xffffffffu, rk);
                int base = 0;
                if (in) base = sc.start[rk];
                if (in) sc.order[base + __popc(peers & lanemask_lt())] = (uint16_t)j;
                __syncwarp();
                if (in && (peers & lanemask_lt()) == 0) sc.start[rk] += __popc(peers);
                __syncwarp();
            }
            // start[] now holds each expert's end; the tasks are order[0 .. je-js)
            const int ns = je - js;
            // ---- expert-major pass
            uint4 xr[VPL], xn[VPL];
            {
                const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)sc.tok[sc.order[0]] * D);
#pragma unroll
                for (int v = 0; v < VPL; ++v) xr[v] = __ldg(src + v * 32 + lane);
            }
            int cur = -1;
            for (int i = 0; i < ns; ++i) {
                const int j = sc.order[i];
                const int k = sc.rank[j];
                if (k != cur) {
                    // expert k's rows: its group is the (k+1)-th committed;
                    // allow S-2 newer groups to stay in flight
                    cp_async_wait<S - 2>();
                    __syncwarp();
                    cur = k;
                    const int kn = k + S - 1;
                    if (kn < n_e) issue(kn, ebase + sc.rlist[kn]);
                    cp_async_commit();
                }
                if (i + 1 < ns) {
                    const uint4 *src =
                        reinterpret_cast<const uint4 *>(x + (size_t)sc.tok[sc.order[i + 1]] * D);
#pragma unroll
                    for (int v = 0; v < VPL; ++v) xn[v] = __ldg(src + v * 32 + lane);
                }
                const uint8_t *slot = ring + (k % S) * Cfg::kPairBytes;
                const uint4 *wr = reinterpret_cast<const uint4 *>(slot);
                const uint4 *vr = reinterpret_cast<const uint4 *>(slot + RB);
                float h = 0.f;
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    float xf[8], wf[8];
                    bf16x8_to_f32(xr[v], xf);
                    bf16x8_to_f32(wr[v * 32 + lane], wf);
#pragma unroll
                    for (int c = 0; c < 8; ++c) h = fmaf(xf[c], wf[c], h);
                }
                h = warp_sum(h);
                const float p = sc.gate[j] * (h / (1.f + __expf(-h)));
                float *yr = y + (size_t)sc.tok[j] * D;
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    float vf[8];
                    bf16x8_to_f32(vr[v * 32 + lane], vf);
                    float *dst = yr + (size_t)(v * 32 + lane) * 8;
                    red_add_v4(dst, p * vf[0], p * vf[1], p * vf[2], p * vf[3]);
                    red_add_v4(dst + 4, p * vf[4], p * vf[5], p * vf[6], p * vf[7]);
                }
                if (i + 1 < ns) {
#pragma unroll
                    for (int v = 0; v < VPL; ++v) xr[v] = xn[v];
                }
            }
            // drain this segment's remaining copies before the ring is reused
            cp_async_wait<0>();
            __syncwarp();
            js = je;
        }
    }
}

template <int VPL>
cudaError_t launch_vpl(const uint16_t *x, const uint16_t *W, const uint16_t *V, const Sizes &sz,
                       const int32_t *tt, const int32_t *te, const float *tg, float *y,
                       int *status, cudaStream_t st) {
    using Cfg = ExpertCfg<VPL>;
    cudaError_t e = cudaFuncSetAttribute(grouped_expert_kernel<VPL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
    if (e != cudaSuccess) return e;
    const int sms = device_sm_count();
    const int64_t warps = (int64_t)sms * Cfg::kWarps;
    int64_t per_warp = (sz.M + warps - 1) / warps;
    if (per_warp < 32) per_warp = 32;
    const int64_t needed = (sz.M + per_warp - 1) / per_warp;          // warps with work
    const int grid = (int)((needed + Cfg::kWarps - 1) / Cfg::kWarps);
    grouped_expert_kernel<VPL><<<grid, Cfg::kThreads, Cfg::kSmem, st>>>(
        x, W, V, sz.L, (int)sz.N, sz.B, (int)sz.M, (int)per_warp, tt, te, tg, y, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_grouped_expert(const uint16_t *x, const uint16_t *W, const uint16_t *V,
                                  const Sizes &sz, const int32_t *task_token,
                                  const int32_t *task_expert, const float *task_gate,
                                  float *y, bool accumulate, void *ws, const WsLayout &lay,
                                  cudaStream_t st) {
    int *status = ws_at<int>(ws, lay.hdr);
    cudaError_t e;
    if (!accumulate) {
        if ((e = cudaMemsetAsync(y, 0, sizeof(float) * (size_t)sz.L * sz.d, st)) != cudaSuccess)
            return e;
    }
    switch (sz.d / 256) {
        case 1: return launch_vpl<1>(x, W, V, sz, task_token, task_expert, task_gate, y, status, st);
        case 2: return launch_vpl<2>(x, W, V, sz, task_token, task_expert, task_gate, y, status, st);
        case 3: return launch_vpl<3>(x, W, V, sz, task_token, task_expert, task_gate, y, status, st);
        case 4: return launch_vpl<4>(x, W, V, sz, task_token, task_expert, task_gate, y, status, st);
        case 5: return launch_vpl<5>(x, W, V, sz, task_token, task_expert, task_gate, y, status, st);
        case 6: return launch_vpl<6>(x, W, V, sz, task_token, task_expert, task_gate, y, status, st);
        case 7: return launch_vpl<7>(x, W, V, sz, task_token, task_expert, task_gate, y, status, st);
        case 8: return launch_vpl<8>(x, W, V, sz, task_token, task_expert, task_gate, y, status, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace omni

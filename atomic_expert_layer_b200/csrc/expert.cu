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
//   1. group pass: P_q = G_q . SiLU(X_q W_q^T) for the task pairs only (G_q is
//      about 8% dense for 4096 tokens over 1.7M experts).  Every warp streams
//      a contiguous share of the sorted tasks (group, token, expert order):
//      per task the expert's W row and the token's x row go through the
//      warp's own cp.async ring (16 bytes per lane, several tasks ahead), and
//      p = g * SiLU(x . w) is written with the expert id into a slot of its
//      token.  A group's experts form one contiguous block of W rows and its
//      tasks are adjacent in the stream, so an expert used by several tokens
//      of the group is read from HBM once and then served by L2.
//   2. token pass: y[t] = sum over the token's slots of p * V[e], one warp
//      per token, V rows through the same kind of ring; y is written once
//      per token.  This is O_q = P_q V_q plus the scatter-add, regrouped by
//      token: on B200 fp32 reductions of per-group partial rows into y
//      (16-byte red.global.add.v4.f32, one L2 sector operation each) ran at
//      about 3 TB/s and cost more than the HBM gather of the rows.
// No kernel here waits on another warp or CTA.
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

constexpr int kChunk = 32;                // tasks whose metadata a warp holds at once

template <int VPL>
struct GateCfg {
    // stages per warp (a stage holds a task's W row and x row).  Measured at
    // d = 1024: many warps with shallow rings beat few warps with deep ones.
    static constexpr int kStages = VPL <= 2 ? 4 : (VPL <= 4 ? 3 : 2);
    static constexpr int kWarps = 4;                      // per CTA; several CTAs per SM
    static constexpr int kRowBytes = 512 * VPL;
    static constexpr int kSmem = kWarps * 2 * kStages * kRowBytes;
};
template <int VPL>
struct CombineCfg {
    static constexpr int kStages = VPL <= 2 ? 4 : 3;
    static constexpr int kWarps = 4;                      // per CTA; several CTAs per SM
    static constexpr int kRowBytes = 512 * VPL;
    static constexpr int kSmem = kWarps * kStages * kRowBytes;
};

// ------------------------------------------------------- 1. group pass
// Warp gw streams the sorted tasks [gw*per_warp, (gw+1)*per_warp): for each
// task the W row of its expert and the x row of its token go through the
// warp's cp.async ring, kStages-1 tasks ahead; p = g * SiLU(x . w) is written
// with the expert id into the token's slot.  Inside a group the tasks of one
// expert are close together, so a repeated W row is normally served by L2.
// Consecutive tasks of one token (a token meets ~1.4 experts per group) load
// and unpack its x row once.  Each lane keeps its partial dot products of 8
// tasks and the warp reduces the 8 together (a transposed butterfly), so the
// reduction costs about one shuffle per task instead of five.
constexpr int kGateBlock = 8;             // tasks reduced together

// bf16 pair (one 32-bit word) -> the two fp32 values, exactly
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// (a0, a1) += (x0, x1) * (w0, w1) as one packed fp32x2 FMA (round to nearest)
__device__ __forceinline__ void fma_f32x2(float &a0, float &a1, float x0, float x1, float w0,
                                          float w1) {
    asm("{\n\t.reg .b64 a, x, w;\n\t"
        "mov.b64 a, {%0, %1};\n\t"
        "mov.b64 x, {%2, %3};\n\t"
        "mov.b64 w, {%4, %5};\n\t"
        "fma.rn.f32x2 a, x, w, a;\n\t"
        "mov.b64 {%0, %1}, a;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "f"(x0), "f"(x1), "f"(w0), "f"(w1));
}

template <int VPL>
__global__ void __launch_bounds__(32 * GateCfg<VPL>::kWarps)
group_gate_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ W, int L, int N,
                  int K, int M, int per_warp, const int32_t *__restrict__ task_token,
                  const int32_t *__restrict__ task_expert, const float *__restrict__ task_gate,
                  int *__restrict__ tok_count, int2 *__restrict__ tok_slots, int *status,
                  const int32_t *__restrict__ group_off, int B, const int32_t *__restrict__ dyn_M) {
    using Cfg = GateCfg<VPL>;
    constexpr int D = 256 * VPL;
    constexpr int S = Cfg::kStages;
    constexpr int RB = Cfg::kRowBytes;
    constexpr int U = kGateBlock;
    static_assert(S - 1 <= kChunk, "prefetch stays within two metadata chunks");
    static_assert(kChunk % U == 0 && U == 8, "blocks of 8 tasks tile a metadata chunk");
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    uint8_t *wring = smem + (size_t)warp * 2 * S * RB;
    uint8_t *xring = wring + S * RB;
    grid_dependency_wait();
    grid_dependents_launch();
    if (dyn_M) {
        // the compacted task list of the tensor-core path: its length is on
        // the device; spread it over every warp of the grid
        M = *dyn_M;
        const int64_t warps = (int64_t)gridDim.x * Cfg::kWarps;
        per_warp = (int)((M + warps - 1) / warps);
        if (per_warp < 1) per_warp = 1;
    }

    const int64_t gw = (int64_t)blockIdx.x * Cfg::kWarps + warp;
    const int64_t a0 = gw * per_warp;
    const int64_t a1 = a0 + per_warp < M ? a0 + per_warp : M;
    if (a0 >= a1) return;
    const int n = (int)(a1 - a0);

    // task metadata of the current chunk of 32 tasks, one task per lane; the
    // slot of each task is claimed here, 32 tasks per atomic round trip
    auto load_meta = [&](int c0, int &t, int &e, float &g, int &slot) {
        const int i = c0 + (int)lane;
        t = 0; e = 0; g = 0.f; slot = K;
        if (i < n) {
            // token order (no schedule): task m is (m / K, idx[m], gate[m])
            t = task_token ? task_token[a0 + i] : (int)((a0 + i) / K);
            e = task_expert[a0 + i];
            g = task_gate[a0 + i];
            if (e < 0 || e >= N || t < 0 || t >= L) {
                set_status(status, OMNI_DEV_BAD_SCHEDULE);
                e = e < 0 || e >= N ? 0 : e;
                t = t < 0 || t >= L ? 0 : t;
            } else if (group_off) {
                // the task must lie in its group's range of the sorted order
                const int q = e / B;
                const int64_t m = a0 + i;
                if (m < group_off[q] || m >= group_off[q + 1]) set_status(status, OMNI_DEV_BAD_SCHEDULE);
            }
            slot = atomicAdd(&tok_count[t], 1);
        }
    };
    int ct, ce, cs, nt, ne, ns;     // current and next chunk (token, expert, slot)
    float cg, ng;
    load_meta(0, ct, ce, cg, cs);
    load_meta(kChunk, nt, ne, ng, ns);
    // Rows of task i into ring slot i % S (rel: its entry in the current
    // (rel < 32) or next (32 <= rel < 64) chunk).  The x row is copied only
    // when the token differs from the previous task's; the consumer makes the
    // same comparison.
    int x_issued = -1;
    auto issue = [&](int i, int rel) {
        const bool same = rel < kChunk;
        const int src = rel % kChunk;
        const int t = __shfl_sync(0xffffffffu, same ? ct : nt, src);
        const int e = __shfl_sync(0xffffffffu, same ? ce : ne, src);
        row_async<VPL>(wring + (i % S) * RB, W + (size_t)e * D, lane);
        if (t != x_issued) {
            row_async<VPL>(xring + (i % S) * RB, x + (size_t)t * D, lane);
            x_issued = t;
        }
    };
#pragma unroll 1
    for (int i = 0; i < S - 1; ++i) {
        if (i < n) issue(i, i);
        cp_async_commit();
    }
    float xf[8 * VPL];              // the current token's x slice, unpacked
    int x_have = -1;
#pragma unroll 1
    for (int base = 0; base < n; base += kChunk) {
        if (base > 0) {             // move to the next chunk of metadata
            ct = nt; ce = ne; cg = ng; cs = ns;
            load_meta(base + kChunk, nt, ne, ng, ns);
        }
#pragma unroll 1
        for (int b0 = 0; b0 < kChunk && base + b0 < n; b0 += U) {
            float hp[U];
#pragma unroll
            for (int j = 0; j < U; ++j) {
                const int i = base + b0 + j;
                hp[j] = 0.f;
                if (i < n) {                               // the same in every lane
                    cp_async_wait<S - 2>();                // task i's rows have landed
                    __syncwarp();
                    const int ip = i + S - 1;
                    if (ip < n) issue(ip, ip - base);
                    cp_async_commit();
                    const int t = __shfl_sync(0xffffffffu, ct, b0 + j);
                    if (t != x_have) {
                        const uint4 *xr = reinterpret_cast<const uint4 *>(xring + (i % S) * RB);
#pragma unroll
                        for (int v = 0; v < VPL; ++v) {
                            const uint4 u = xr[v * 32 + lane];
                            const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                xf[8 * v + 2 * q] = bf_lo(wd[q]);
                                xf[8 * v + 2 * q + 1] = bf_hi(wd[q]);
                            }
                        }
                        x_have = t;
                    }
                    const uint4 *wr = reinterpret_cast<const uint4 *>(wring + (i % S) * RB);
                    float c0 = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f;
#pragma unroll
                    for (int v = 0; v < VPL; ++v) {
                        const uint4 u = wr[v * 32 + lane];
                        fma_f32x2(c0, c1, xf[8 * v + 0], xf[8 * v + 1], bf_lo(u.x), bf_hi(u.x));
                        fma_f32x2(c2, c3, xf[8 * v + 2], xf[8 * v + 3], bf_lo(u.y), bf_hi(u.y));
                        fma_f32x2(c0, c1, xf[8 * v + 4], xf[8 * v + 5], bf_lo(u.z), bf_hi(u.z));
                        fma_f32x2(c2, c3, xf[8 * v + 6], xf[8 * v + 7], bf_lo(u.w), bf_hi(u.w));
                    }
                    hp[j] = (c0 + c1) + (c2 + c3);
                }
            }
            // Transposed butterfly: after the three exchanges lane l holds
            // the sum over lanes l ^ {4, 8, 16} of task (l >> 2) & 7's
            // partials; two more exchanges add lanes l ^ {1, 2}.
            {
                const bool up = (lane & 16u) != 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float send = up ? hp[k] : hp[k + 4];
                    const float keep = up ? hp[k + 4] : hp[k];
                    hp[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
                }
            }
            {
                const bool up = (lane & 8u) != 0;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float send = up ? hp[k] : hp[k + 2];
                    const float keep = up ? hp[k + 2] : hp[k];
                    hp[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
                }
            }
            float h;
            {
                const bool up = (lane & 4u) != 0;
                const float send = up ? hp[0] : hp[1];
                const float keep = up ? hp[1] : hp[0];
                h = keep + __shfl_xor_sync(0xffffffffu, send, 4);
            }
            h += __shfl_xor_sync(0xffffffffu, h, 2);
            h += __shfl_xor_sync(0xffffffffu, h, 1);
            const int jt = (int)((lane >> 2) & 7u);
            const int src = b0 + jt;
            const int t = __shfl_sync(0xffffffffu, ct, src);
            const int e = __shfl_sync(0xffffffffu, ce, src);
            const float g = __shfl_sync(0xffffffffu, cg, src);
            const int slot = __shfl_sync(0xffffffffu, cs, src);
            if ((lane & 3u) == 0 && base + src < n) {
                const float p = g * (h / (1.f + __expf(-h)));
                if (slot < K)
                    tok_slots[(size_t)t * K + slot] = make_int2(e, __float_as_int(p));
                else
                    set_status(status, OMNI_DEV_BAD_SCHEDULE);
            }
        }
    }
    cp_async_wait<0>();
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
    grid_dependency_wait();
    grid_dependents_launch();
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

// ------------------------------------------------- 2b. token pass, split
// Small batches: one CTA per token, its slots dealt round-robin to kSplit
// warps (slot w, w + kSplit, ...), so a token's V rows are fetched kSplit at
// a time instead of one warp walking all K.  Each warp's partial row goes to
// shared memory (reusing the row rings once every copy has landed) and the
// CTA adds the kSplit partials in a fixed order and writes y once.
constexpr int kSplit = 8;

template <int VPL>
struct SplitCfg {
    static constexpr int kStages = 3;
    static constexpr int kRowBytes = 512 * VPL;
    static constexpr int kRing = kSplit * kStages * kRowBytes;
    static constexpr int kPart = kSplit * 256 * VPL * 4;        // fp32 partial rows
    static constexpr int kSmem = kRing > kPart ? kRing : kPart;
};

template <int VPL>
__global__ void __launch_bounds__(32 * kSplit)
token_split_kernel(const uint16_t *__restrict__ V, int L, int N, int K,
                   const int *__restrict__ tok_count, const int2 *__restrict__ tok_slots,
                   float *__restrict__ y, int accumulate, int *status) {
    using Cfg = SplitCfg<VPL>;
    constexpr int D = 256 * VPL;
    constexpr int S = Cfg::kStages;
    constexpr int RB = Cfg::kRowBytes;
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    uint8_t *ring = smem + (size_t)warp * S * RB;
    grid_dependency_wait();
    grid_dependents_launch();
    const int t = blockIdx.x;
    if (t >= L) return;                                  // the same in every thread
    int n = tok_count[t];
    if (n > K) {
        set_status(status, OMNI_DEV_BAD_SCHEDULE);
        n = K;
    }
    const int2 *sl = tok_slots + (size_t)t * K;
    const int nw = n > warp ? (n - warp + kSplit - 1) / kSplit : 0;   // this warp's slots
    // (expert, p) of this warp's slots j, j < 32 per block: slot warp + kSplit * j
    auto load_block = [&](int j0) {
        const int j = j0 + (int)lane;
        int2 v = j < nw ? sl[warp + kSplit * j] : make_int2(0, 0);
        if (v.x < 0 || v.x >= N) v.x = 0;
        return v;
    };
    int2 mine = load_block(0);
    float acc[VPL * 8];
#pragma unroll
    for (int c = 0; c < VPL * 8; ++c) acc[c] = 0.f;
#pragma unroll
    for (int j = 0; j < S - 1; ++j) {
        if (j < nw) {
            const int e = __shfl_sync(0xffffffffu, mine.x, j);
            row_async<VPL>(ring + (j % S) * RB, V + (size_t)e * D, lane);
        }
        cp_async_commit();
    }
    for (int j = 0; j < nw; ++j) {
        cp_async_wait<S - 2>();
        __syncwarp();
        const float p = __int_as_float(__shfl_sync(0xffffffffu, mine.y, j & 31));
        const int jn = j + S - 1;
        if (jn < nw) {
            int en;
            if ((jn >> 5) == (j >> 5)) {
                en = __shfl_sync(0xffffffffu, mine.x, jn & 31);
            } else {
                const int2 nx = sl[warp + kSplit * jn];
                en = (nx.x < 0 || nx.x >= N) ? 0 : nx.x;
            }
            row_async<VPL>(ring + (jn % S) * RB, V + (size_t)en * D, lane);
        }
        cp_async_commit();
        const uint4 *vr = reinterpret_cast<const uint4 *>(ring + (j % S) * RB);
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            float vf[8];
            bf16x8_to_f32(vr[v * 32 + lane], vf);
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[8 * v + c] = fmaf(p, vf[c], acc[8 * v + c]);
        }
        if (((j + 1) & 31) == 0 && j + 1 < nw) mine = load_block(j + 1);
    }
    cp_async_wait<0>();
    __syncthreads();                                     // every ring is idle: reuse as partials
    float *part = reinterpret_cast<float *>(smem) + (size_t)warp * D;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        float4 *dst = reinterpret_cast<float4 *>(part + (size_t)(v * 32 + lane) * 8);
        dst[0] = make_float4(acc[8 * v], acc[8 * v + 1], acc[8 * v + 2], acc[8 * v + 3]);
        dst[1] = make_float4(acc[8 * v + 4], acc[8 * v + 5], acc[8 * v + 6], acc[8 * v + 7]);
    }
    __syncthreads();
    const float *P = reinterpret_cast<const float *>(smem);
    float *yr = y + (size_t)t * D;
    for (int i = (int)threadIdx.x * 4; i < D; i += 32 * kSplit * 4) {
        float4 r = reinterpret_cast<const float4 *>(P + i)[0];
#pragma unroll
        for (int w = 1; w < kSplit; ++w) {
            const float4 q = reinterpret_cast<const float4 *>(P + (size_t)w * D + i)[0];
            r.x += q.x; r.y += q.y; r.z += q.z; r.w += q.w;
        }
        float4 *dst = reinterpret_cast<float4 *>(yr + i);
        if (accumulate) {
            const float4 o = dst[0];
            r.x += o.x; r.y += o.y; r.z += o.z; r.w += o.w;
        }
        dst[0] = r;
    }
}

template <int VPL>
cudaError_t launch_vpl(const uint16_t *x, const uint16_t *W, const uint16_t *V, const Sizes &sz,
                       const int32_t *tt, const int32_t *te, const float *tg, float *y,
                       bool accumulate, int *tok_count, int2 *tok_slots, int *status,
                       cudaStream_t st, const int32_t *group_off, const int32_t *dyn_M) {
    using G = GateCfg<VPL>;
    using C = CombineCfg<VPL>;
    cudaError_t e = cudaFuncSetAttribute(group_gate_kernel<VPL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, G::kSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(token_combine_kernel<VPL>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(token_split_kernel<VPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SplitCfg<VPL>::kSmem);
    if (e != cudaSuccess) return e;
    const int sms = device_sm_count();
    {
        int per_sm = (227 * 1024) / G::kSmem;
        if (per_sm < 1) per_sm = 1;
        if (per_sm > 16) per_sm = 16;
        const int64_t warps = (int64_t)sms * per_sm * G::kWarps;
        // small batches spread down to one task per warp (latency, not issue, bounds them)
        const int64_t per_warp = (sz.M + warps - 1) / warps;
        const int64_t needed = (sz.M + per_warp - 1) / per_warp;      // warps with work
        const int grid = (int)((needed + G::kWarps - 1) / G::kWarps);
        e = launch(group_gate_kernel<VPL>, dim3(grid), dim3(32 * G::kWarps), G::kSmem, st, x, W,
                   sz.L, (int)sz.N, sz.K, (int)sz.M, (int)per_warp, tt, te, tg, tok_count,
                   tok_slots, status, group_off, sz.B, dyn_M);
        if (e != cudaSuccess) return e;
    }
    if (sz.L <= 4 * sms) {
        // few tokens: one CTA of kSplit warps per token
        e = launch(token_split_kernel<VPL>, dim3((unsigned)sz.L), dim3(32 * kSplit),
                   (size_t)SplitCfg<VPL>::kSmem, st, V, sz.L, (int)sz.N, sz.K,
                   (const int *)tok_count, (const int2 *)tok_slots, y, accumulate ? 1 : 0,
                   status);
    } else {
        int per_sm = (227 * 1024) / C::kSmem;
        if (per_sm < 1) per_sm = 1;
        if (per_sm > 16) per_sm = 16;
        int64_t grid = (int64_t)sms * per_sm;
        const int64_t need = (sz.L + C::kWarps - 1) / C::kWarps;
        if (grid > need) grid = need;
        e = launch(token_combine_kernel<VPL>, dim3((unsigned)grid), dim3(32 * C::kWarps), C::kSmem,
                   st, V, sz.L, (int)sz.N, sz.K, (const int *)tok_count,
                   (const int2 *)tok_slots, y, accumulate ? 1 : 0, status);
    }
    return e;
}

}  // namespace

cudaError_t launch_grouped_expert(const uint16_t *x, const uint16_t *W, const uint16_t *V,
                                  const Sizes &sz, const int32_t *task_token,
                                  const int32_t *task_expert, const float *task_gate,
                                  float *y, bool accumulate, void *ws, const WsLayout &lay,
                                  cudaStream_t st, const int32_t *group_offsets,
                                  const int32_t *dyn_M) {
    int *status = ws_at<int>(ws, lay.hdr);
    int *tok_count = ws_at<int>(ws, lay.tok_count);
    int2 *tok_slots = ws_at<int2>(ws, lay.tok_slots);
    switch (sz.d / 256) {
#define OMNI_CASE(n) \
        case n: return launch_vpl<n>(x, W, V, sz, task_token, task_expert, task_gate, y, accumulate, \
                                     tok_count, tok_slots, status, st, group_offsets, dyn_M);
        OMNI_CASE(1) OMNI_CASE(2) OMNI_CASE(3) OMNI_CASE(4)
        OMNI_CASE(5) OMNI_CASE(6) OMNI_CASE(7) OMNI_CASE(8)
#undef OMNI_CASE
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace omni

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
// 1.7M experts), so the kernel computes only the task pairs, on CUDA cores,
// and spends its effort on keeping HBM busy:
//   - persistent CTAs (one per SM) claim work items from a device counter;
//     an item is a group, or a slice of at most kItemTasks tasks of one;
//   - warp 0 (producer) finds the item's distinct experts (bitmap over B),
//     splits them into chunks that fit a ring of shared-memory row slots, and
//     issues one bulk copy per W row and per V row (cp.async.bulk, L2
//     evict-first; rows are read once), signalling an mbarrier per chunk;
//   - the other warps (consumers) take the item's token runs (consecutive
//     tasks of one token; the schedule orders a group by token) round-robin:
//     load x_t once, and for each task of the run whose expert is in the
//     chunk compute h = x_t . w_e (warp reduction), p = g * SiLU(h) and
//     accumulate p * v_e in registers; then one vector reduction (red.add.v4)
//     per 4 columns into y[t], which is L2-resident for typical L.
// Every mbarrier wait is bounded; on timeout the status word records
// OMNI_DEV_WAIT_TIMEOUT, the producer waits (bounded) for its own copies and
// the CTA returns.
#include "omni_common.cuh"
#include "omni_internal.h"

namespace omni {
namespace {

constexpr int kNChunk = 6;                 // chunk metadata ring
constexpr int kSmemBudget = 227 * 1024;    // opt-in shared memory per CTA

struct ChunkMeta {
    int q;           // group
    int m0;          // first task of the item
    int ntask;       // tasks in the item
    int n_e;         // experts in this chunk; -1 = end of work
    int c0;          // rank of the chunk's first expert among the item's experts
    int slot0;       // ring slot of the chunk's first expert
    int n_runs;      // token runs of the item
    int pad;
    uint16_t rank[kItemTasks];          // per task: rank of its expert in the item
    uint16_t run_start[kItemTasks + 1]; // per run: first task (relative to m0)
    float gate[kItemTasks];
    int run_token[kItemTasks];
};

struct ProducerScratch {
    uint32_t bitmap[OMNI_MAX_B / 32];
    int word_prefix[OMNI_MAX_B / 32];
    uint16_t rlist[OMNI_MAX_B];
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &u, float *f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// --------------------------------------------------------------- items
// One CTA of 1024 threads turns the active groups into work items
// {q, m_begin, m_end} of at most kItemTasks tasks, and resets the claim counter.
__global__ void __launch_bounds__(1024) build_items_kernel(
    const int32_t *__restrict__ group_offsets, const int32_t *__restrict__ active_groups,
    const int32_t *__restrict__ num_active_p, int64_t G, int64_t M, int64_t max_items,
    int4 *__restrict__ items, WsHeader *hdr) {
    __shared__ int sh[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int na = *num_active_p;
    if (na < 0 || na > G) {
        if (tid == 0) set_status(&hdr->status, OMNI_DEV_BAD_SCHEDULE);
        na = 0;
    }
    const int per = (na + 1023) / 1024;
    const int a0 = tid * per;
    const int a1 = a0 + per < na ? a0 + per : na;
    int cnt = 0;
    for (int a = a0; a < a1; ++a) {
        const int q = active_groups[a];
        if (q < 0 || q >= G) continue;
        const int m0 = group_offsets[q], m1 = group_offsets[q + 1];
        if (m0 < 0 || m1 > M || m1 < m0) continue;
        const int n = m1 - m0;
        if (n > 0) cnt += (n + kItemTasks - 1) / kItemTasks;
    }
    const int incl = warp_iscan(cnt);
    if (lane == 31) sh[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int s = sh[lane];
        const int is = warp_iscan(s);
        sh[lane] = is - s;
        if (lane == 31) {
            hdr->total_items = (int)(is < max_items ? is : max_items);
            hdr->item_counter = 0;
            if (is > max_items) set_status(&hdr->status, OMNI_DEV_BAD_SCHEDULE);
        }
    }
    __syncthreads();
    int pos = sh[warp] + incl - cnt;
    for (int a = a0; a < a1; ++a) {
        const int q = active_groups[a];
        if (q < 0 || q >= G) {
            set_status(&hdr->status, OMNI_DEV_BAD_SCHEDULE);
            continue;
        }
        const int m0 = group_offsets[q], m1 = group_offsets[q + 1];
        if (m0 < 0 || m1 > M || m1 < m0) {
            set_status(&hdr->status, OMNI_DEV_BAD_SCHEDULE);
            continue;
        }
        for (int m = m0; m < m1; m += kItemTasks) {
            if (pos < max_items)
                items[pos] = make_int4(q, m, m + kItemTasks < m1 ? m + kItemTasks : m1, 0);
            ++pos;
        }
    }
}

// ---------------------------------------------------------- main kernel
template <int VPL>
struct ExpertCfg {
    static constexpr int kD = 256 * VPL;                 // d
    static constexpr int kRowBytes = 2 * kD;             // one bf16 row
    static constexpr int kSlotBytes = 2 * kRowBytes;     // W row + V row
    static constexpr int kConsumers = VPL <= 4 ? 16 : 8; // consumer warps
    static constexpr int kThreads = 32 * (1 + kConsumers);
    static constexpr int kFixed = ((int)(sizeof(ChunkMeta) * kNChunk + sizeof(ProducerScratch) +
                                         16 * kNChunk + 1023) / 1024) * 1024;
    static constexpr int kNSlot = (kSmemBudget - kFixed) / kSlotBytes;
    static constexpr int kMaxChunk = kNSlot / 2;         // experts per chunk
    static constexpr int kSmem = kFixed + kNSlot * kSlotBytes;
    static_assert(kNSlot >= 8, "ring too small");
};

template <int VPL>
__global__ void __launch_bounds__(ExpertCfg<VPL>::kThreads, 1)
grouped_expert_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ W,
                      const uint16_t *__restrict__ V, int L, int N, int B,
                      const int32_t *__restrict__ task_token,
                      const int32_t *__restrict__ task_expert,
                      const float *__restrict__ task_gate, const int4 *__restrict__ items,
                      float *__restrict__ y, WsHeader *hdr) {
    using Cfg = ExpertCfg<VPL>;
    constexpr int D = Cfg::kD;
    constexpr int NSLOT = Cfg::kNSlot;
    constexpr int RB = Cfg::kRowBytes;
    extern __shared__ __align__(1024) uint8_t smem[];
    // slots first (1024-aligned), then metadata
    uint8_t *slots = smem;
    ChunkMeta *meta = reinterpret_cast<ChunkMeta *>(smem + (size_t)NSLOT * Cfg::kSlotBytes);
    ProducerScratch *ps = reinterpret_cast<ProducerScratch *>(meta + kNChunk);
    uint64_t *full = reinterpret_cast<uint64_t *>(ps + 1);
    uint64_t *empty = full + kNChunk;

    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    int *status = &hdr->status;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNChunk; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], Cfg::kConsumers);
        }
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ============================ producer ============================
        const uint64_t pol = l2_evict_first_policy();
        const int total = *(volatile int *)&hdr->total_items;
        const int nwords = (B + 31) >> 5;
        int seq = 0, oldest = 0;
        long long head = 0, freed = 0;
        bool ok = true;
        while (ok) {
            int it = 0;
            if (lane == 0) it = atomicAdd(&hdr->item_counter, 1);
            it = __shfl_sync(0xffffffffu, it, 0);
            if (it >= total) break;
            const int4 item = items[it];
            const int q = item.x, m0 = item.y, ntask = item.z - item.y;
            const int64_t ebase = (int64_t)q * B;
            // distinct experts of the item, as ranks in ascending expert id
            for (int w = lane; w < nwords; w += 32) ps->bitmap[w] = 0u;
            __syncwarp();
            for (int j = lane; j < ntask; j += 32) {
                int r = (int)(task_expert[m0 + j] - ebase);
                if (r < 0 || r >= B || ebase + r >= N) {
                    set_status(status, OMNI_DEV_BAD_SCHEDULE);
                    r = 0;
                }
                atomicOr(&ps->bitmap[r >> 5], 1u << (r & 31));
            }
            __syncwarp();
            const uint32_t wbits = lane < (unsigned)nwords ? ps->bitmap[lane] : 0u;
            const int cnt = __popc(wbits);
            const int incl = warp_iscan(cnt);
            const int n_dist = __shfl_sync(0xffffffffu, incl, 31);
            if (lane < (unsigned)nwords) {
                ps->word_prefix[lane] = incl - cnt;
                uint32_t bits = wbits;
                int pos = incl - cnt;
                while (bits) {
                    const int b = __ffs(bits) - 1;
                    ps->rlist[pos++] = (uint16_t)(lane * 32 + b);
                    bits &= bits - 1;
                }
            }
            __syncwarp();
            for (int c0 = 0; c0 < n_dist && ok; c0 += Cfg::kMaxChunk) {
                const int n_e = n_dist - c0 < Cfg::kMaxChunk ? n_dist - c0 : Cfg::kMaxChunk;
                // reserve a metadata entry and n_e ring slots
                while (seq - oldest >= kNChunk || head + n_e - freed > NSLOT) {
                    const int so = oldest % kNChunk;
                    if (!mbar_wait(&empty[so], (uint32_t)((oldest / kNChunk) & 1), status)) {
                        ok = false;
                        break;
                    }
                    freed += meta[so].n_e;
                    ++oldest;
                }
                if (!ok) break;
                const int s = seq % kNChunk;
                ChunkMeta &m = meta[s];
                // per-task data and token runs of the item (same for every chunk)
                int nrun = 0;
                for (int j0 = 0; j0 < ntask; j0 += 32) {
                    const int j = j0 + (int)lane;
                    int tok = -1;
                    bool start = false;
                    if (j < ntask) {
                        int r = (int)(task_expert[m0 + j] - ebase);
                        if (r < 0 || r >= B) r = 0;
                        const int wd = r >> 5;
                        m.rank[j] = (uint16_t)(ps->word_prefix[wd] +
                                               __popc(ps->bitmap[wd] & ((1u << (r & 31)) - 1u)));
                        m.gate[j] = task_gate[m0 + j];
                        tok = task_token[m0 + j];
                        if (tok < 0 || tok >= L) {
                            set_status(status, OMNI_DEV_BAD_SCHEDULE);
                            tok = 0;
                        }
                        start = (j == 0) || (task_token[m0 + j - 1] != task_token[m0 + j]);
                    }
                    const unsigned bal = __ballot_sync(0xffffffffu, start);
                    if (start) {
                        const int pos = nrun + __popc(bal & lanemask_lt());
                        m.run_start[pos] = (uint16_t)j;
                        m.run_token[pos] = tok;
                    }
                    nrun += __popc(bal);
                }
                if (lane == 0) {
                    m.q = q;
                    m.m0 = m0;
                    m.ntask = ntask;
                    m.n_e = n_e;
                    m.c0 = c0;
                    m.slot0 = (int)(head % NSLOT);
                    m.n_runs = nrun;
                    m.run_start[nrun] = (uint16_t)ntask;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(n_e * 2 * RB));
                __syncwarp();
                for (int i = lane; i < n_e; i += 32) {
                    const int slot = (int)((head + i) % NSLOT);
                    const int64_t e = ebase + ps->rlist[c0 + i];
                    uint8_t *dst = slots + (size_t)slot * Cfg::kSlotBytes;
                    bulk_g2s(dst, W + e * D, RB, &full[s], pol);
                    bulk_g2s(dst + RB, V + e * D, RB, &full[s], pol);
                }
                head += n_e;
                ++seq;
                __syncwarp();
            }
        }
        if (ok) {
            // end-of-work marker for the consumers
            while (seq - oldest >= kNChunk) {
                const int so = oldest % kNChunk;
                if (!mbar_wait(&empty[so], (uint32_t)((oldest / kNChunk) & 1), status)) {
                    ok = false;
                    break;
                }
                ++oldest;
            }
            if (ok) {
                const int s = seq % kNChunk;
                if (lane == 0) {
                    meta[s].n_e = -1;
                    mbar_arrive(&full[s]);
                }
                ++seq;
            }
        }
        if (!ok) {
            // never leave bulk copies in flight: wait (bounded) for every
            // chunk that was issued and not released
            for (int c = oldest; c < seq; ++c) {
                mbar_wait(&full[c % kNChunk], (uint32_t)((c / kNChunk) & 1), status);
            }
        }
        return;
    }

    // =============================== consumers ===============================
    const int cw = warp - 1;
    int seq = 0;
    while (true) {
        const int s = seq % kNChunk;
        if (!mbar_wait(&full[s], (uint32_t)((seq / kNChunk) & 1), status)) break;
        const ChunkMeta &m = meta[s];
        const int n_e = m.n_e;
        if (n_e < 0) break;
        const int c0 = m.c0, slot0 = m.slot0, nrun = m.n_runs;
        for (int run = cw; run < nrun; run += Cfg::kConsumers) {
            const int j0 = m.run_start[run], j1 = m.run_start[run + 1];
            const int t = m.run_token[run];
            float acc[VPL * 8];
#pragma unroll
            for (int i = 0; i < VPL * 8; ++i) acc[i] = 0.f;
            float xf[VPL * 8];
            bool any = false;
            for (int j = j0; j < j1; ++j) {
                const int li = (int)m.rank[j] - c0;
                if ((unsigned)li >= (unsigned)n_e) continue;
                if (!any) {
                    const uint4 *xr = reinterpret_cast<const uint4 *>(x + (size_t)t * D);
#pragma unroll
                    for (int v = 0; v < VPL; ++v) bf16x8_to_f32(__ldg(xr + v * 32 + lane), xf + 8 * v);
                    any = true;
                }
                int slot = slot0 + li;
                if (slot >= NSLOT) slot -= NSLOT;
                const uint4 *wr = reinterpret_cast<const uint4 *>(slots + (size_t)slot * Cfg::kSlotBytes);
                const uint4 *vr = reinterpret_cast<const uint4 *>(slots + (size_t)slot * Cfg::kSlotBytes + RB);
                float h = 0.f;
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    float wf[8];
                    bf16x8_to_f32(wr[v * 32 + lane], wf);
#pragma unroll
                    for (int i = 0; i < 8; ++i) h = fmaf(xf[8 * v + i], wf[i], h);
                }
                h = warp_sum(h);
                const float p = m.gate[j] * (h / (1.f + __expf(-h)));
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    float vf[8];
                    bf16x8_to_f32(vr[v * 32 + lane], vf);
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[8 * v + i] = fmaf(p, vf[i], acc[8 * v + i]);
                }
            }
            if (any) {
                float *yr = y + (size_t)t * D;
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    float *dst = yr + (size_t)(v * 32 + lane) * 8;
                    red_add_v4(dst, acc[8 * v], acc[8 * v + 1], acc[8 * v + 2], acc[8 * v + 3]);
                    red_add_v4(dst + 4, acc[8 * v + 4], acc[8 * v + 5], acc[8 * v + 6], acc[8 * v + 7]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        ++seq;
    }
}

template <int VPL>
cudaError_t launch_vpl(const uint16_t *x, const uint16_t *W, const uint16_t *V, const Sizes &sz,
                       const int32_t *tt, const int32_t *te, const float *tg, const int4 *items,
                       float *y, WsHeader *hdr, cudaStream_t st) {
    using Cfg = ExpertCfg<VPL>;
    cudaError_t e = cudaFuncSetAttribute(grouped_expert_kernel<VPL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
    if (e != cudaSuccess) return e;
    const int grid = device_sm_count();
    grouped_expert_kernel<VPL><<<grid, Cfg::kThreads, Cfg::kSmem, st>>>(
        x, W, V, sz.L, (int)sz.N, sz.B, tt, te, tg, items, y, hdr);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_grouped_expert(const uint16_t *x, const uint16_t *W, const uint16_t *V,
                                  const Sizes &sz, const int32_t *task_token,
                                  const int32_t *task_expert, const float *task_gate,
                                  const int32_t *group_offsets, const int32_t *active_groups,
                                  const int32_t *num_active, float *y, bool accumulate,
                                  void *ws, const WsLayout &lay, cudaStream_t st) {
    WsHeader *hdr = ws_at<WsHeader>(ws, lay.hdr);
    int4 *items = ws_at<int4>(ws, lay.items);
    cudaError_t e;
    if (!accumulate) {
        if ((e = cudaMemsetAsync(y, 0, sizeof(float) * (size_t)sz.L * sz.d, st)) != cudaSuccess)
            return e;
    }
    build_items_kernel<<<1, 1024, 0, st>>>(group_offsets, active_groups, num_active, sz.G, sz.M,
                                           sz.max_items, items, hdr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    switch (sz.d / 256) {
        case 1: return launch_vpl<1>(x, W, V, sz, task_token, task_expert, task_gate, items, y, hdr, st);
        case 2: return launch_vpl<2>(x, W, V, sz, task_token, task_expert, task_gate, items, y, hdr, st);
        case 3: return launch_vpl<3>(x, W, V, sz, task_token, task_expert, task_gate, items, y, hdr, st);
        case 4: return launch_vpl<4>(x, W, V, sz, task_token, task_expert, task_gate, items, y, hdr, st);
        case 5: return launch_vpl<5>(x, W, V, sz, task_token, task_expert, task_gate, items, y, hdr, st);
        case 6: return launch_vpl<6>(x, W, V, sz, task_token, task_expert, task_gate, items, y, hdr, st);
        case 7: return launch_vpl<7>(x, W, V, sz, task_token, task_expert, task_gate, items, y, hdr, st);
        case 8: return launch_vpl<8>(x, W, V, sz, task_token, task_expert, task_gate, items, y, hdr, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace omni

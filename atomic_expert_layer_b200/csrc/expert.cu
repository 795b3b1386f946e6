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
//   - work items are fixed ranges of kItemTasks tasks of the sorted task
//     array; persistent CTAs (one per SM) take items b, b + grid, ... so no
//     work list or claim counter is needed.  An item is cut where the group
//     changes; a group cut by an item boundary loads the experts common to
//     both halves twice (about one row per boundary);
//   - warp 0 (producer) holds the next item's tasks in registers while it
//     issues the current one, finds each group segment's distinct experts
//     (bitmap over B), splits them into chunks that fit a ring of shared-
//     memory row slots, publishes the chunk's description (meta_full) and
//     issues one bulk copy per W row and per V row (cp.async.bulk, L2
//     evict-first; rows are read once), completing on data_full;
//   - the other warps (consumers) take the segment's token runs (consecutive
//     tasks of one token; the schedule orders a group by token) round-robin.
//     A consumer requests the x row of its run as soon as the chunk is
//     described, then for each task of the run whose expert is in the chunk
//     computes h = x_t . w_e (warp reduction), p = g * SiLU(h) and
//     accumulates p * v_e in registers; then one vector reduction (red.add.v4)
//     per 4 columns into y[t], which is L2-resident for typical L.
// Every mbarrier wait is bounded; on timeout the status word records
// OMNI_DEV_WAIT_TIMEOUT, the producer waits (bounded) for its own copies and
// the CTA returns.
#include "omni_common.cuh"
#include "omni_internal.h"

namespace omni {
namespace {

constexpr int kNChunk = 8;                 // chunk metadata ring
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
    uint16_t seg_start[kItemTasks + 2];
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &u, float *f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// ---------------------------------------------------------- main kernel
template <int VPL>
struct ExpertCfg {
    static constexpr int kD = 256 * VPL;                 // d
    static constexpr int kRowBytes = 2 * kD;             // one bf16 row
    static constexpr int kSlotBytes = 2 * kRowBytes;     // W row + V row
    static constexpr int kConsumers = VPL <= 2 ? 16 : (VPL <= 4 ? 12 : 6);  // consumer warps
    static constexpr int kThreads = 32 * (1 + kConsumers);
    // after the slots: chunk metadata, producer scratch, then the barriers on
    // a 16-byte boundary (mbarriers need 8-byte alignment)
    static constexpr int kMetaBytes = (int)(sizeof(ChunkMeta) * kNChunk);
    static constexpr int kBarOff = ((kMetaBytes + (int)sizeof(ProducerScratch) + 15) / 16) * 16;
    static constexpr int kFixed = ((kBarOff + 3 * 8 * kNChunk + 1023) / 1024) * 1024;
    static constexpr int kNSlot = (kSmemBudget - kFixed) / kSlotBytes;
    static constexpr int kMaxChunk = kNSlot / 2;         // experts per chunk
    static constexpr int kSmem = kFixed + kNSlot * kSlotBytes;
    static_assert(kNSlot >= 8, "ring too small");
    static_assert((kNSlot * kSlotBytes) % 1024 == 0, "slots keep 1 KB alignment");
    static_assert((kNSlot * kSlotBytes + kBarOff) % 16 == 0, "barriers 16-byte aligned");
};
static_assert(sizeof(ChunkMeta) % 4 == 0, "metadata entries stay 4-byte aligned");

constexpr int kTPL = kItemTasks / 32;                    // tasks per producer lane

template <int VPL>
__global__ void __launch_bounds__(ExpertCfg<VPL>::kThreads, 1)
grouped_expert_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ W,
                      const uint16_t *__restrict__ V, int L, int N, int B, int M,
                      const int32_t *__restrict__ task_token,
                      const int32_t *__restrict__ task_expert,
                      const float *__restrict__ task_gate, float *__restrict__ y,
                      WsHeader *hdr) {
    using Cfg = ExpertCfg<VPL>;
    constexpr int D = Cfg::kD;
    constexpr int NSLOT = Cfg::kNSlot;
    constexpr int RB = Cfg::kRowBytes;
    extern __shared__ __align__(1024) uint8_t smem[];
    // slots first, then chunk metadata, producer scratch and barriers
    uint8_t *slots = smem;
    uint8_t *fixed = smem + (size_t)NSLOT * Cfg::kSlotBytes;
    ChunkMeta *meta = reinterpret_cast<ChunkMeta *>(fixed);
    ProducerScratch *ps = reinterpret_cast<ProducerScratch *>(fixed + Cfg::kMetaBytes);
    uint64_t *meta_full = reinterpret_cast<uint64_t *>(fixed + Cfg::kBarOff);   // chunk described
    uint64_t *data_full = meta_full + kNChunk;                    // its rows have landed
    uint64_t *empty = data_full + kNChunk;                        // consumers are done

    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    int *status = &hdr->status;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNChunk; ++s) {
            mbar_init(&meta_full[s], 1);
            mbar_init(&data_full[s], 1);
            mbar_init(&empty[s], Cfg::kConsumers);
        }
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ============================ producer ============================
        // Items are fixed ranges of kItemTasks sorted tasks, CTA b taking
        // items b, b + grid, ...  The next item's tasks are loaded into
        // registers while the current one is being issued.
        const uint64_t pol = l2_evict_first_policy();
        const int nitems = (M + kItemTasks - 1) / kItemTasks;
        const int nwords = (B + 31) >> 5;
        int seq = 0, oldest = 0;
        long long head = 0, freed = 0;
        bool ok = true;

        // next item's tasks, loaded one item ahead
        int pe[kTPL], pt[kTPL];
        float pg[kTPL];
#define OMNI_PREFETCH_ITEM(ITEM)                                                  \
    _Pragma("unroll") for (int u = 0; u < kTPL; ++u) {                            \
        const int m_ = (ITEM) * kItemTasks + u * 32 + (int)lane;                  \
        const bool v_ = (ITEM) < nitems && m_ < M;                                \
        pe[u] = v_ ? __ldg(task_expert + m_) : -1;                                \
        pt[u] = v_ ? __ldg(task_token + m_) : -1;                                 \
        pg[u] = v_ ? __ldg(task_gate + m_) : 0.f;                                 \
    }
        int item = blockIdx.x;
        OMNI_PREFETCH_ITEM(item);
        for (; item < nitems && ok; item += gridDim.x) {
            int ce[kTPL], ct[kTPL], cq[kTPL];
            float cg[kTPL];
#pragma unroll
            for (int u = 0; u < kTPL; ++u) {
                ce[u] = pe[u];
                ct[u] = pt[u];
                cg[u] = pg[u];
            }
            OMNI_PREFETCH_ITEM(item + gridDim.x);
            const int m0 = item * kItemTasks;
            const int ntask = min(kItemTasks, M - m0);
            // validate, split into groups (segments): q changes along the item
            int nseg = 0;
#pragma unroll
            for (int u = 0; u < kTPL; ++u) {
                const int j = u * 32 + (int)lane;
                int e = ce[u], t = ct[u];
                if (j < ntask) {
                    if (e < 0 || e >= N) {
                        set_status(status, OMNI_DEV_BAD_SCHEDULE);
                        e = 0;
                    }
                    if (t < 0 || t >= L) {
                        set_status(status, OMNI_DEV_BAD_SCHEDULE);
                        t = 0;
                    }
                }
                ce[u] = e;
                ct[u] = t;
                cq[u] = j < ntask ? e / B : -1;
                int prevq = __shfl_up_sync(0xffffffffu, cq[u], 1);
                if (u > 0) {
                    const int last = __shfl_sync(0xffffffffu, cq[u - 1], 31);
                    if (lane == 0) prevq = last;
                }
                const bool start = j < ntask && (j == 0 || prevq != cq[u]);
                const unsigned bal = __ballot_sync(0xffffffffu, start);
                if (start) ps->seg_start[nseg + __popc(bal & lanemask_lt())] = (uint16_t)j;
                nseg += __popc(bal);
            }
            if (lane == 0) ps->seg_start[nseg] = (uint16_t)ntask;
            __syncwarp();
            for (int sg = 0; sg < nseg && ok; ++sg) {
                const int js = ps->seg_start[sg], je = ps->seg_start[sg + 1];
                // the group of the segment: q of task js
                int qv = 0;
#pragma unroll
                for (int u = 0; u < kTPL; ++u) qv |= (u * 32 + (int)lane == js) ? cq[u] : 0;
                const int q = __reduce_or_sync(0xffffffffu, (unsigned)qv);
                const int64_t ebase = (int64_t)q * B;
                // distinct experts of the segment, ranked by expert id
                for (int w = lane; w < nwords; w += 32) ps->bitmap[w] = 0u;
                __syncwarp();
#pragma unroll
                for (int u = 0; u < kTPL; ++u) {
                    const int j = u * 32 + (int)lane;
                    if (j >= js && j < je) {
                        const int r = (int)(ce[u] - ebase);
                        atomicOr(&ps->bitmap[r >> 5], 1u << (r & 31));
                    }
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
                    const int n_e = min(n_dist - c0, Cfg::kMaxChunk);
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
                    // per task of the segment: expert rank, gate; token runs
                    int nrun = 0;
#pragma unroll
                    for (int u = 0; u < kTPL; ++u) {
                        const int j = u * 32 + (int)lane;
                        const bool in = j >= js && j < je;
                        int prevt = __shfl_up_sync(0xffffffffu, ct[u], 1);
                        if (u > 0) {
                            const int last = __shfl_sync(0xffffffffu, ct[u - 1], 31);
                            if (lane == 0) prevt = last;
                        }
                        if (in) {
                            const int r = (int)(ce[u] - ebase);
                            const int wd = r >> 5;
                            m.rank[j - js] = (uint16_t)(ps->word_prefix[wd] +
                                                        __popc(ps->bitmap[wd] & ((1u << (r & 31)) - 1u)));
                            m.gate[j - js] = cg[u];
                        }
                        const bool start = in && (j == js || prevt != ct[u]);
                        const unsigned bal = __ballot_sync(0xffffffffu, start);
                        if (start) {
                            const int pos = nrun + __popc(bal & lanemask_lt());
                            m.run_start[pos] = (uint16_t)(j - js);
                            m.run_token[pos] = ct[u];
                        }
                        nrun += __popc(bal);
                    }
                    if (lane == 0) {
                        m.q = q;
                        m.m0 = m0 + js;
                        m.ntask = je - js;
                        m.n_e = n_e;
                        m.c0 = c0;
                        m.slot0 = (int)(head % NSLOT);
                        m.n_runs = nrun;
                        m.run_start[nrun] = (uint16_t)(je - js);
                    }
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&meta_full[s]);
                        mbar_arrive_expect_tx(&data_full[s], (uint32_t)(n_e * 2 * RB));
                    }
                    __syncwarp();
                    for (int i = lane; i < n_e; i += 32) {
                        const int slot = (int)((head + i) % NSLOT);
                        const int64_t e = ebase + ps->rlist[c0 + i];
                        uint8_t *dst = slots + (size_t)slot * Cfg::kSlotBytes;
                        bulk_g2s(dst, W + e * D, RB, &data_full[s], pol);
                        bulk_g2s(dst + RB, V + e * D, RB, &data_full[s], pol);
                    }
                    head += n_e;
                    ++seq;
                    __syncwarp();
                }
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
                    mbar_arrive(&meta_full[s]);
                }
                ++seq;
            }
        }
#undef OMNI_PREFETCH_ITEM
        if (!ok) {
            // never leave bulk copies in flight: wait (bounded) for every
            // chunk that was issued and not released
            for (int c = oldest; c < seq; ++c)
                mbar_wait(&data_full[c % kNChunk], (uint32_t)((c / kNChunk) & 1), status);
        }
        return;
    }

    // =============================== consumers ===============================
    // Each consumer warp takes runs cw, cw + kConsumers, ... of every chunk.
    // The x row of its first run is requested as soon as the chunk is
    // described, before its expert rows have landed.
    const int cw = warp - 1;
    int seq = 0;
    while (true) {
        const int s = seq % kNChunk;
        const uint32_t par = (uint32_t)((seq / kNChunk) & 1);
        if (!mbar_wait(&meta_full[s], par, status)) break;
        const ChunkMeta &m = meta[s];
        const int n_e = m.n_e;
        if (n_e < 0) break;
        const int c0 = m.c0, slot0 = m.slot0, nrun = m.n_runs;
        uint4 xr[VPL];
        int run = cw;
        if (run < nrun) {
            const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)m.run_token[run] * D);
#pragma unroll
            for (int v = 0; v < VPL; ++v) xr[v] = __ldg(src + v * 32 + lane);
        }
        if (!mbar_wait(&data_full[s], par, status)) break;
        for (; run < nrun; run += Cfg::kConsumers) {
            const int j0 = m.run_start[run], j1 = m.run_start[run + 1];
            const int t = m.run_token[run];
            // next run's x row, requested before this run's arithmetic
            uint4 xn[VPL];
            const int nxt = run + Cfg::kConsumers;
            if (nxt < nrun) {
                const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)m.run_token[nxt] * D);
#pragma unroll
                for (int v = 0; v < VPL; ++v) xn[v] = __ldg(src + v * 32 + lane);
            }
            float acc[VPL * 8];
#pragma unroll
            for (int i = 0; i < VPL * 8; ++i) acc[i] = 0.f;
            bool any = false;
            for (int j = j0; j < j1; ++j) {
                const int li = (int)m.rank[j] - c0;
                if ((unsigned)li >= (unsigned)n_e) continue;
                any = true;
                int slot = slot0 + li;
                if (slot >= NSLOT) slot -= NSLOT;
                const uint4 *wr = reinterpret_cast<const uint4 *>(slots + (size_t)slot * Cfg::kSlotBytes);
                const uint4 *vr = reinterpret_cast<const uint4 *>(slots + (size_t)slot * Cfg::kSlotBytes + RB);
                float h = 0.f;
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    float xf[8], wf[8];
                    bf16x8_to_f32(xr[v], xf);
                    bf16x8_to_f32(wr[v * 32 + lane], wf);
#pragma unroll
                    for (int i = 0; i < 8; ++i) h = fmaf(xf[i], wf[i], h);
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
            if (nxt < nrun) {
#pragma unroll
                for (int v = 0; v < VPL; ++v) xr[v] = xn[v];
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        ++seq;
    }
}

template <int VPL>
cudaError_t launch_vpl(const uint16_t *x, const uint16_t *W, const uint16_t *V, const Sizes &sz,
                       const int32_t *tt, const int32_t *te, const float *tg, float *y,
                       WsHeader *hdr, cudaStream_t st) {
    using Cfg = ExpertCfg<VPL>;
    cudaError_t e = cudaFuncSetAttribute(grouped_expert_kernel<VPL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
    if (e != cudaSuccess) return e;
    const int64_t nitems = (sz.M + kItemTasks - 1) / kItemTasks;
    const int sms = device_sm_count();
    const int grid = (int)(nitems < sms ? nitems : sms);
    grouped_expert_kernel<VPL><<<grid, Cfg::kThreads, Cfg::kSmem, st>>>(
        x, W, V, sz.L, (int)sz.N, sz.B, (int)sz.M, tt, te, tg, y, hdr);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_grouped_expert(const uint16_t *x, const uint16_t *W, const uint16_t *V,
                                  const Sizes &sz, const int32_t *task_token,
                                  const int32_t *task_expert, const float *task_gate,
                                  float *y, bool accumulate, void *ws, const WsLayout &lay,
                                  cudaStream_t st) {
    WsHeader *hdr = ws_at<WsHeader>(ws, lay.hdr);
    cudaError_t e;
    if (!accumulate) {
        if ((e = cudaMemsetAsync(y, 0, sizeof(float) * (size_t)sz.L * sz.d, st)) != cudaSuccess)
            return e;
    }
    switch (sz.d / 256) {
        case 1: return launch_vpl<1>(x, W, V, sz, task_token, task_expert, task_gate, y, hdr, st);
        case 2: return launch_vpl<2>(x, W, V, sz, task_token, task_expert, task_gate, y, hdr, st);
        case 3: return launch_vpl<3>(x, W, V, sz, task_token, task_expert, task_gate, y, hdr, st);
        case 4: return launch_vpl<4>(x, W, V, sz, task_token, task_expert, task_gate, y, hdr, st);
        case 5: return launch_vpl<5>(x, W, V, sz, task_token, task_expert, task_gate, y, hdr, st);
        case 6: return launch_vpl<6>(x, W, V, sz, task_token, task_expert, task_gate, y, hdr, st);
        case 7: return launch_vpl<7>(x, W, V, sz, task_token, task_expert, task_gate, y, hdr, st);
        case 8: return launch_vpl<8>(x, W, V, sz, task_token, task_expert, task_gate, y, hdr, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace omni

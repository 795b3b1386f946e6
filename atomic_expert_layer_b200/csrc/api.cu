// api.cu -- the C ABI of libomni (declared in include/omni.h): argument
// checks, workspace layout and the order of kernel launches.  No allocation,
// no host synchronisation except in omni_get_device_status.
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cstring>

#include "omni_common.cuh"
#include "omni_internal.h"
#include "sched_token.cuh"

namespace omni {

namespace {
constexpr int kVersion = 1;
constexpr int kTokenOrderMaxL = 16;   // decode batches skip the schedule (see omni.h)

inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
}  // namespace

int device_sm_count() {
    // filled once per device; several host threads may race to fill an entry,
    // and all of them store the same value
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

bool make_sizes(int L, int d, int N_r, int N_c, int K, int B, Sizes *sz) {
    if (L <= 0 || d <= 0 || N_r <= 0 || N_c <= 0 || K <= 0 || B <= 0) return false;
    sz->L = L; sz->d = d; sz->N_r = N_r; sz->N_c = N_c; sz->K = K; sz->B = B;
    sz->N = (int64_t)N_r * N_c;
    sz->M = (int64_t)L * K;
    sz->G = (sz->N + B - 1) / B;
    sz->Kr = K < N_r ? K : N_r;
    sz->Kc = K < N_c ? K : N_c;
    sz->C = merge_candidates(K, sz->Kr, sz->Kc);
    sz->ntiles = (sz->M + kSortTile - 1) / kSortTile;
    int nbits = 0;
    while (nbits < 31 && ((int64_t)1 << nbits) < sz->G) ++nbits;
    sz->qbits = nbits;
    sz->passes = (nbits + 7) / 8;
    return true;
}

void set_dense(Sizes *sz, unsigned flags) {
    sz->dense = false;
    sz->dense_thr = 0;
    sz->dense_cap = 0;
    if (flags & OMNI_EXPERT_SPARSE) return;
    // By default the tensor-core path is considered only for large expert
    // stages (tasks x width >= 2^31): its fixed cost (six more launches) is
    // then a small share of the stage, and below that size an expert rarely
    // reaches the threshold.
    const bool want = (flags & OMNI_EXPERT_DENSE) || sz->M * (int64_t)sz->d >= ((int64_t)1 << 31);
    if (!want) return;
    // An expert joins the tile GEMMs when >= thr tasks use it: its column
    // costs 4 L d tensor-core flops, against a gathered W and V row per task
    // on the CUDA-core path (break-even near L / 96 tasks at d = 2048).
    int thr = (sz->L + 95) / 96;
    if (thr < 32) thr = 32;
    int64_t most = sz->M / thr;                  // experts that can reach thr
    if (most > sz->N) most = sz->N;
    if (most == 0) return;
    int64_t cap = (most + 255) / 256 * 256;
    if (cap > 4096) cap = 4096;
    // G (fp32) and P (bf16) take 6 bytes per token and column: at most 768 MB
    while (cap > 256 && 6 * (int64_t)sz->L * cap > ((int64_t)768 << 20)) cap -= 256;
    sz->dense = true;
    sz->dense_thr = thr;
    sz->dense_cap = (int)cap;
}

WsLayout make_layout(const Sizes &sz, unsigned regions) {
    WsLayout w;
    std::memset(&w, 0, sizeof w);
    size_t o = 0;
    auto take = [&](size_t bytes) { const size_t at = o; o = align256(o + bytes); return at; };
    const size_t L = (size_t)sz.L, M = (size_t)sz.M, G = (size_t)sz.G;
    w.hdr = take(sizeof(WsHeader));
    // counters that must be zero when a call starts: right after the header
    if (regions & kRegSched) {
        w.z_cnt = take(4 * G);
        w.z_ndist = take(4);
        w.bitmap = take(4 * (size_t)((sz.N + 31) / 32));
        w.hist = take(4 * 256 * (size_t)sz.ntiles * (size_t)sz.passes);   // one per radix pass
    }
    if (regions & kRegExpert) {
        w.tok_count = take(4 * L);
    }
    const bool dense = (regions & kRegDense) && sz.dense;
    if (dense) {
        w.dz_cnt = take(4 * (size_t)sz.N);
        w.dz_ghot = take(4 * (G + 1));
        w.dz_ccount = take(8);
    }
    w.zero_end = o;
    if (regions & kRegExpert) w.dec_bar = take(8);      // outside the zeroed prefix
    if (regions & kRegRouter) {
        w.s_r = take(4 * L * sz.N_r);
        w.s_c = take(4 * L * sz.N_c);
        w.part_r = take(8 * L * 2 * (size_t)((sz.N_r + 2 * kGemmPartCols - 1) / (2 * kGemmPartCols)));
        w.part_c = take(8 * L * 2 * (size_t)((sz.N_c + 2 * kGemmPartCols - 1) / (2 * kGemmPartCols)));
        w.flags = take(4 * 2 * L);
        w.row_val = take(4 * L * sz.Kr);
        w.row_idx = take(4 * L * sz.Kr);
        w.col_val = take(4 * L * sz.Kc);
        w.col_idx = take(4 * L * sz.Kc);
        w.idx = take(4 * L * sz.K);
        w.score = take(4 * L * sz.K);
        w.gate = take(4 * L * sz.K);
    }
    if (regions & kRegSched) {
        w.a_tok = take(4 * M); w.a_exp = take(4 * M); w.a_gate = take(4 * M);
        w.b_tok = take(4 * M); w.b_exp = take(4 * M); w.b_gate = take(4 * M);
    }
    if (regions & kRegSchedOut) {
        w.t_tok = take(4 * M); w.t_exp = take(4 * M); w.t_gate = take(4 * M);
        w.g_off = take(4 * (G + 1));
        w.g_cnt = take(4 * G);
        w.g_act = take(4 * G);
        w.n_act = take(4);
        w.n_dist = take(4);
    }
    if (regions & kRegExpert) w.tok_slots = take(8 * M);
    if (dense) {
        const size_t cap = (size_t)sz.dense_cap, d = (size_t)sz.d;
        w.d_ehot = take(4);
        w.d_list = take(4 * cap);
        w.d_whot = take(2 * cap * d);
        w.d_vt = take(2 * d * cap);
        w.d_G = take(4 * L * cap);
        w.d_P = take(2 * L * cap);
        w.d_ctok = take(4 * M);
        w.d_cexp = take(4 * M);
        w.d_cgate = take(4 * M);
    }
    w.total = o;
    return w;
}

namespace {
// One CTA waits on a barrier that never completes; the bounded wait gives up.
__global__ void selftest_wait_kernel(int *status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_limit(&bar, 0u, status, limit_ns);
}
}  // namespace

}  // namespace omni

using namespace omni;

namespace {

int check_common(int L, int d, int N_r, int N_c, int K, int B, bool router, Sizes *sz) {
    if (!make_sizes(L, d, N_r, N_c, K, B, sz)) return OMNI_ERR_INVALID_ARG;
    if ((int64_t)K > sz->N) return OMNI_ERR_INVALID_ARG;
    if (sz->M > INT_MAX || sz->N > INT_MAX) return OMNI_ERR_UNSUPPORTED;
    if (K > OMNI_MAX_K || B > OMNI_MAX_B) return OMNI_ERR_UNSUPPORTED;
    if (router && (N_r > OMNI_MAX_AXIS || N_c > OMNI_MAX_AXIS)) return OMNI_ERR_UNSUPPORTED;
    return OMNI_OK;
}

int check_ws(const Sizes &sz, unsigned regions, void *ws, size_t ws_bytes, WsLayout *lay) {
    if (!ws) return OMNI_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return OMNI_ERR_INVALID_ARG;
    *lay = make_layout(sz, regions);
    if (ws_bytes < lay->total) return OMNI_ERR_WORKSPACE;
    return OMNI_OK;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? OMNI_OK : OMNI_ERR_CUDA; }

// Clears the status word and the counters the call's kernels accumulate into.
int reset_workspace(void *ws, const WsLayout &lay, cudaStream_t st) {
    first_launch_in_call();             // the next kernel follows this memset
    return cuda_rc(cudaMemsetAsync(ws, 0, lay.zero_end, st));
}

int router_topk_impl(const uint16_t *x, const uint16_t *W_r, const uint16_t *W_c,
                     const Sizes &sz, float *p_r, float *p_c, int32_t *idx, float *score,
                     float *gate, unsigned flags, void *ws, const WsLayout &lay,
                     cudaStream_t st, const SchedPrep *prep = nullptr) {
    int *status = ws_at<int>(ws, lay.hdr);
    float *row_val = ws_at<float>(ws, lay.row_val), *col_val = ws_at<float>(ws, lay.col_val);
    int *row_idx = ws_at<int>(ws, lay.row_idx), *col_idx = ws_at<int>(ws, lay.col_idx);
    int *row_flags = ws_at<int>(ws, lay.flags);
    const float *dead_r = nullptr, *dead_c = nullptr;
    cudaError_t e;
    if (flags & OMNI_ROUTER_LOGPROBS_IN) {
        e = launch_axis_topk(p_r, p_c, false, nullptr, nullptr, nullptr, nullptr, sz.L, sz.N_r,
                             sz.N_c, sz.K, row_val, row_idx, col_val, col_idx, row_flags, status, st);
    } else {
        float *s_r = ws_at<float>(ws, lay.s_r), *s_c = ws_at<float>(ws, lay.s_c);
        float *part_r = ws_at<float>(ws, lay.part_r), *part_c = ws_at<float>(ws, lay.part_c);
        if (router_small_ok(sz.L, sz.d)) {
            // a handful of tokens: streamed projection, LogSoftmax in the axis kernels
            e = launch_router_small(x, W_r, W_c, sz.L, sz.d, sz.N_r, sz.N_c, s_r, s_c, st);
            part_r = part_c = nullptr;
        } else {
            e = launch_router_gemm(x, W_r, W_c, sz.L, sz.d, sz.N_r, sz.N_c, s_r, s_c, part_r,
                                   part_c, status, st);
        }
        if (e != cudaSuccess) return OMNI_ERR_CUDA;
        e = launch_axis_topk(s_r, s_c, true, part_r, part_c, p_r, p_c, sz.L, sz.N_r, sz.N_c,
                             sz.K, row_val, row_idx, col_val, col_idx, row_flags, status, st);
        // the logits are dead after the axis kernels; large ones are dropped
        // from L2 unwritten (small ones cost more to drop than to keep)
        if ((size_t)4 * sz.L * (sz.N_r + sz.N_c) >= ((size_t)16 << 20)) {
            dead_r = s_r;
            dead_c = s_c;
        }
    }
    if (e != cudaSuccess) return OMNI_ERR_CUDA;
    e = launch_merge_topk(row_val, row_idx, col_val, col_idx, sz.L, sz.N_c, sz.K, sz.Kr, sz.Kc,
                          sz.C, idx, score, gate, dead_r, dead_c, sz.N_r, prep, st);
    return cuda_rc(e);
}

// The expert stage on a sorted schedule.  With the tensor-core path, the
// dense experts' tasks go through the tile GEMMs (which add into y after
// the CUDA-core passes wrote it) and the rest through the CUDA-core passes.
cudaError_t expert_stage(const uint16_t *x, const uint16_t *W, const uint16_t *V, const Sizes &sz,
                         const int32_t *tt, const int32_t *te, const float *tg,
                         const int32_t *goff, const int32_t *gact, const int32_t *nact, float *y,
                         bool accumulate, void *ws, const WsLayout &lay, cudaStream_t st,
                         bool check_offsets) {
    if (!sz.dense)
        return launch_grouped_expert(x, W, V, sz, tt, te, tg, y, accumulate, ws, lay, st,
                                     check_offsets ? goff : nullptr);
    int *status = ws_at<int>(ws, lay.hdr);
    const DenseWs o = dense_ws_of(sz, ws, lay);
    cudaError_t e = launch_dense_prepare(W, V, sz, tt, te, tg, goff, gact, nact, o, status, st);
    if (e != cudaSuccess) return e;
    e = launch_grouped_expert(x, W, V, sz, o.c_tok, o.c_exp, o.c_gate, y, accumulate, ws, lay, st,
                              nullptr, o.ccount);
    if (e != cudaSuccess) return e;
    return launch_dense_gemms(x, sz, o, y, status, st);
}

}  // namespace

extern "C" {

int omni_version(void) { return kVersion; }

const char *omni_status_string(int s) {
    switch (s) {
        case OMNI_OK: return "OMNI_OK";
        case OMNI_ERR_INVALID_ARG: return "OMNI_ERR_INVALID_ARG";
        case OMNI_ERR_UNSUPPORTED: return "OMNI_ERR_UNSUPPORTED";
        case OMNI_ERR_WORKSPACE: return "OMNI_ERR_WORKSPACE";
        case OMNI_ERR_CUDA: return "OMNI_ERR_CUDA";
        case OMNI_ERR_DEVICE: return "OMNI_ERR_DEVICE";
        default: return "unknown omni_status";
    }
}

const char *omni_device_status_string(int s) {
    switch (s) {
        case OMNI_DEV_OK: return "OMNI_DEV_OK";
        case OMNI_DEV_BAD_EXPERT: return "OMNI_DEV_BAD_EXPERT";
        case OMNI_DEV_WAIT_TIMEOUT: return "OMNI_DEV_WAIT_TIMEOUT";
        case OMNI_DEV_BAD_SCHEDULE: return "OMNI_DEV_BAD_SCHEDULE";
        default: return "unknown device status";
    }
}

size_t omni_workspace_size_flags(int L, int d, int N_r, int N_c, int K, int B, unsigned flags) {
    Sizes sz;
    if (check_common(L, d, N_r, N_c, K, B, true, &sz) != OMNI_OK) return 0;
    if (flags & OMNI_TOKEN_ORDER) return make_layout(sz, kRegRouter | kRegExpert).total;
    set_dense(&sz, flags);
    return make_layout(sz, kRegAll).total;
}

size_t omni_workspace_size(int L, int d, int N_r, int N_c, int K, int B) {
    return omni_workspace_size_flags(L, d, N_r, N_c, K, B, 0u);
}

size_t omni_router_workspace_size(int L, int N_r, int N_c, int K) {
    Sizes sz;
    if (check_common(L, 8, N_r, N_c, K, 1, true, &sz) != OMNI_OK) return 0;
    return make_layout(sz, kRegRouter).total;
}

size_t omni_schedule_workspace_size(int L, int K, int N, int B) {
    Sizes sz;
    if (N <= 0 || check_common(L, 8, N, 1, K, B, false, &sz) != OMNI_OK) return 0;
    return make_layout(sz, kRegSched).total;
}

size_t omni_expert_workspace_size_flags(int L, int d, int K, int N, int B, unsigned flags) {
    Sizes sz;
    if (N <= 0 || check_common(L, d, N, 1, K, B, false, &sz) != OMNI_OK) return 0;
    set_dense(&sz, flags);
    return make_layout(sz, kRegExpert | kRegDense).total;
}

size_t omni_expert_workspace_size(int L, int d, int K, int N, int B) {
    return omni_expert_workspace_size_flags(L, d, K, N, B, 0u);
}

int omni_router_topk(const omni_bf16 *x, const omni_bf16 *W_r, const omni_bf16 *W_c, int L,
                     int d, int N_r, int N_c, int K, float *p_r, float *p_c, int32_t *idx,
                     float *score, float *gate, unsigned flags, void *ws, size_t ws_bytes,
                     omni_stream_t stream) {
    const bool lp_in = (flags & OMNI_ROUTER_LOGPROBS_IN) != 0;
    Sizes sz;
    int rc = check_common(L, lp_in ? 8 : d, N_r, N_c, K, 1, true, &sz);
    if (rc) return rc;
    if (!p_r || !p_c || !idx || !score || !gate) return OMNI_ERR_INVALID_ARG;
    if (!lp_in) {
        if (!x || !W_r || !W_c) return OMNI_ERR_INVALID_ARG;
        if (d % 8 != 0) return OMNI_ERR_UNSUPPORTED;
        if (!aligned16(x) || !aligned16(W_r) || !aligned16(W_c)) return OMNI_ERR_INVALID_ARG;
    }
    if (!aligned4(p_r) || !aligned4(p_c)) return OMNI_ERR_INVALID_ARG;
    WsLayout lay;
    if ((rc = check_ws(sz, kRegRouter, ws, ws_bytes, &lay))) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (flags & OMNI_TOPK_BLOCKWISE) {
        // the pages' blockwise grid top-K, on caller log-probabilities; its
        // candidates use the logits area (s_r, s_c), idle in this mode
        if (!lp_in || blockwise_bands(N_r, N_c, K) < 1) return OMNI_ERR_UNSUPPORTED;
        if ((rc = reset_workspace(ws, lay, st))) return rc;
        return cuda_rc(launch_topk_blockwise(p_r, p_c, L, N_r, N_c, K, ws_at<void>(ws, lay.s_r),
                                             idx, score, gate, st));
    }
    if ((rc = reset_workspace(ws, lay, st))) return rc;
    return router_topk_impl(x, W_r, W_c, sz, p_r, p_c, idx, score, gate, flags, ws, lay, st);
}

int omni_schedule(const int32_t *idx, const float *gate, int L, int K, int N, int B,
                  int32_t *task_token, int32_t *task_expert, float *task_gate,
                  int32_t *group_offsets, int32_t *group_counts, int32_t *active_groups,
                  int32_t *num_active, int32_t *num_distinct, void *ws, size_t ws_bytes,
                  omni_stream_t stream) {
    if (N <= 0) return OMNI_ERR_INVALID_ARG;
    Sizes sz;
    int rc = check_common(L, 8, N, 1, K, B, false, &sz);   // an N x 1 grid gives the same N
    if (rc) return rc;
    if (!idx || !gate || !task_token || !task_expert || !task_gate || !group_offsets ||
        !group_counts || !active_groups || !num_active || !num_distinct)
        return OMNI_ERR_INVALID_ARG;
    WsLayout lay;
    if ((rc = check_ws(sz, kRegSched, ws, ws_bytes, &lay))) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = reset_workspace(ws, lay, st))) return rc;
    return cuda_rc(launch_schedule(idx, gate, sz, task_token, task_expert, task_gate,
                                   group_offsets, group_counts, active_groups, num_active,
                                   num_distinct, ws, lay, st));
}

int omni_grouped_expert_fwd(const omni_bf16 *x, const omni_bf16 *W, const omni_bf16 *V, int L,
                            int d, int K, int N, int B, const int32_t *task_token,
                            const int32_t *task_expert, const float *task_gate,
                            const int32_t *group_offsets, const int32_t *active_groups,
                            const int32_t *num_active, float *y, unsigned flags, void *ws,
                            size_t ws_bytes, omni_stream_t stream) {
    if (N <= 0) return OMNI_ERR_INVALID_ARG;
    Sizes sz;
    int rc = check_common(L, d, N, 1, K, B, false, &sz);
    if (rc) return rc;
    if (!x || !W || !V || !task_token || !task_expert || !task_gate || !group_offsets ||
        !active_groups || !num_active || !y)
        return OMNI_ERR_INVALID_ARG;
    if (d % 256 != 0 || d > OMNI_MAX_D) return OMNI_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(W) || !aligned16(V) || !aligned16(y))
        return OMNI_ERR_INVALID_ARG;
    set_dense(&sz, flags);
    WsLayout lay;
    if ((rc = check_ws(sz, kRegExpert | kRegDense, ws, ws_bytes, &lay))) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = reset_workspace(ws, lay, st))) return rc;
    return cuda_rc(expert_stage(x, W, V, sz, task_token, task_expert, task_gate, group_offsets,
                                active_groups, num_active, y, (flags & OMNI_Y_ACCUMULATE) != 0,
                                ws, lay, st, /*check_offsets=*/true));
}

int omni_routed_fwd(const omni_bf16 *x, const omni_bf16 *W, const omni_bf16 *V,
                    const omni_bf16 *W_r, const omni_bf16 *W_c, int L, int d, int N_r, int N_c,
                    int K, int B, float *y, int32_t *idx_out, float *gate_out, unsigned flags,
                    void *ws, size_t ws_bytes, omni_stream_t stream) {
    Sizes sz;
    int rc = check_common(L, d, N_r, N_c, K, B, true, &sz);
    if (rc) return rc;
    if (!x || !W || !V || !W_r || !W_c || !y) return OMNI_ERR_INVALID_ARG;
    if (d % 256 != 0 || d > OMNI_MAX_D) return OMNI_ERR_UNSUPPORTED;
    if (flags & OMNI_TOPK_BLOCKWISE) return OMNI_ERR_UNSUPPORTED;   // router_topk only
    if (!aligned16(x) || !aligned16(W) || !aligned16(V) || !aligned16(W_r) || !aligned16(W_c) ||
        !aligned16(y))
        return OMNI_ERR_INVALID_ARG;
    const bool token_order = (flags & OMNI_TOKEN_ORDER) || L <= kTokenOrderMaxL;
    if (!token_order) set_dense(&sz, flags);
    WsLayout lay;
    if ((rc = check_ws(sz, token_order ? (unsigned)(kRegRouter | kRegExpert) : (unsigned)kRegAll,
                       ws, ws_bytes, &lay)))
        return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool fused = L <= kTokenOrderMaxL && decode_fused_ok(L, d, N_r, N_c, K, sz.Kr, sz.Kc, sz.C);
    // the fused step clears its own status word and needs no zeroed counters
    if (!fused && (rc = reset_workspace(ws, lay, st))) return rc;
    int32_t *idx = ws_at<int32_t>(ws, lay.idx);
    float *score = ws_at<float>(ws, lay.score), *gate = ws_at<float>(ws, lay.gate);
    // scheduled path: the merge kernel also runs the schedule's per-token step;
    // nothing here reads the distinct-expert count, so it is not kept
    SchedPrep prep = sched_prep_of(sz, ws, lay);
    prep.bitmap = nullptr;
    // the expert stage needs each group's tasks together, in no particular
    // order inside the group: no radix pass, so no first-pass digit counts
    if (sched_unordered(sz)) {
        prep.hist0 = nullptr;
        prep.unordered = 1;
    }
    if (fused) {
        // a handful of tokens: the whole step in one cooperative launch
        static std::atomic<unsigned> epochs{0};
        unsigned epoch = ++epochs;
        if (epoch == 0) epoch = ++epochs;
        rc = cuda_rc(launch_decode_fused(
            x, W, V, W_r, W_c, L, d, N_r, N_c, K, sz.Kr, sz.Kc, sz.C, ws_at<float>(ws, lay.s_r),
            ws_at<float>(ws, lay.s_c), ws_at<float>(ws, lay.row_val), ws_at<int>(ws, lay.row_idx),
            ws_at<float>(ws, lay.col_val), ws_at<int>(ws, lay.col_idx), idx, score, gate, y,
            (flags & OMNI_Y_ACCUMULATE) != 0, ws_at<unsigned long long>(ws, lay.dec_bar), epoch,
            ws_at<int>(ws, lay.hdr), st));
        if (rc) return rc;
        if (idx_out && (rc = cuda_rc(cudaMemcpyAsync(idx_out, idx, 4 * (size_t)sz.M,
                                                     cudaMemcpyDeviceToDevice, st))))
            return rc;
        if (gate_out && (rc = cuda_rc(cudaMemcpyAsync(gate_out, gate, 4 * (size_t)sz.M,
                                                      cudaMemcpyDeviceToDevice, st))))
            return rc;
        return OMNI_OK;
    }
    rc = router_topk_impl(x, W_r, W_c, sz, nullptr, nullptr, idx, score, gate,
                          flags & ~OMNI_ROUTER_LOGPROBS_IN, ws, lay, st,
                          token_order ? nullptr : &prep);
    if (rc) return rc;
    if (token_order) {
        // tasks in token order, read straight from the routing (no schedule)
        if ((rc = cuda_rc(launch_grouped_expert(x, W, V, sz, nullptr, idx, gate, y,
                                                (flags & OMNI_Y_ACCUMULATE) != 0, ws, lay, st))))
            return rc;
    } else {
        int32_t *tt = ws_at<int32_t>(ws, lay.t_tok), *te = ws_at<int32_t>(ws, lay.t_exp);
        float *tg = ws_at<float>(ws, lay.t_gate);
        int32_t *goff = ws_at<int32_t>(ws, lay.g_off), *gcnt = ws_at<int32_t>(ws, lay.g_cnt);
        int32_t *gact = ws_at<int32_t>(ws, lay.g_act), *nact = ws_at<int32_t>(ws, lay.n_act);
        int32_t *ndist = ws_at<int32_t>(ws, lay.n_dist);
        if ((rc = cuda_rc(launch_schedule(idx, gate, sz, tt, te, tg, goff, gcnt, gact, nact,
                                          ndist, ws, lay, st, /*prepared=*/true,
                                          /*any_order=*/true))))
            return rc;
        if ((rc = cuda_rc(expert_stage(x, W, V, sz, tt, te, tg, goff, gact, nact, y,
                                       (flags & OMNI_Y_ACCUMULATE) != 0, ws, lay, st,
                                       /*check_offsets=*/false))))
            return rc;
    }
    if (idx_out &&
        (rc = cuda_rc(cudaMemcpyAsync(idx_out, idx, 4 * (size_t)sz.M, cudaMemcpyDeviceToDevice, st))))
        return rc;
    if (gate_out &&
        (rc = cuda_rc(cudaMemcpyAsync(gate_out, gate, 4 * (size_t)sz.M, cudaMemcpyDeviceToDevice, st))))
        return rc;
    return OMNI_OK;
}

int omni_routed_bwd(const omni_bf16 *x, const omni_bf16 *W, const omni_bf16 *V,
                    const omni_bf16 *W_r, const omni_bf16 *W_c, int L, int d, int N_r, int N_c,
                    int K, const int32_t *idx, const float *gate, const float *dy, float *dx,
                    float *dW, float *dV, float *dW_r, float *dW_c, unsigned flags, void *ws,
                    size_t ws_bytes, omni_stream_t stream) {
    Sizes sz;
    int rc = check_common(L, d, N_r, N_c, K, 1, true, &sz);
    if (rc) return rc;
    if (flags != 0) return OMNI_ERR_INVALID_ARG;
    if (!x || !W || !V || !W_r || !W_c || !idx || !gate || !dy || !dx || !dW || !dV || !dW_r ||
        !dW_c || !ws)
        return OMNI_ERR_INVALID_ARG;
    if (d % 256 != 0 || d > OMNI_MAX_D) return OMNI_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(W) || !aligned16(V) || !aligned16(W_r) || !aligned16(W_c) ||
        !aligned16(dy) || !aligned16(dx) || !aligned16(dW) || !aligned16(dV) ||
        !aligned16(dW_r) || !aligned16(dW_c))
        return OMNI_ERR_INVALID_ARG;
    if (ws_bytes < sizeof(WsHeader) || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return OMNI_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    first_launch_in_call();
    // with room for them: two bitmaps over the experts (seen, used more than
    // once), then per router row a pair counter and kBwdRowCap (token, ds) slots
    const size_t map = align256(4 * (size_t)((sz.N + 31) / 32));
    const size_t nrows = (size_t)sz.N_r + sz.N_c;
    const size_t cnt_bytes = align256(4 * nrows);
    const size_t marks_end = sizeof(WsHeader) + 2 * map;
    const size_t rows_end = marks_end + cnt_bytes + 8 * nrows * kBwdRowCap;
    const bool marks = ws_bytes >= marks_end;
    const bool rows = ws_bytes >= rows_end;
    const size_t clear = rows ? marks_end + cnt_bytes : (marks ? marks_end : sizeof(WsHeader));
    if (cudaMemsetAsync(ws, 0, clear, st) != cudaSuccess) return OMNI_ERR_CUDA;
    uint32_t *seen = marks ? ws_at<uint32_t>(ws, sizeof(WsHeader)) : nullptr;
    uint32_t *shared_rows = marks ? ws_at<uint32_t>(ws, sizeof(WsHeader) + map) : nullptr;
    int *rcnt = rows ? ws_at<int>(ws, marks_end) : nullptr;
    int2 *rslots = rows ? ws_at<int2>(ws, marks_end + cnt_bytes) : nullptr;
    return cuda_rc(launch_routed_bwd(x, W, V, W_r, W_c, sz, idx, gate, dy, dx, dW, dV, dW_r,
                                     dW_c, seen, shared_rows, rcnt, rslots, kBwdRowCap,
                                     ws_at<int>(ws, 0), st));
}

size_t omni_routed_bwd_workspace_size(int L, int d, int N_r, int N_c, int K) {
    Sizes sz;
    if (check_common(L, d, N_r, N_c, K, 1, true, &sz)) return 0;
    const size_t nrows = (size_t)sz.N_r + sz.N_c;
    return sizeof(WsHeader) + 2 * align256(4 * (size_t)((sz.N + 31) / 32)) +
           align256(4 * nrows) + 8 * nrows * kBwdRowCap;
}

size_t omni_shared_mlp_workspace_size(int L, int d, int F) {
    if (L <= 0 || d <= 0 || F <= 0) return 0;
    return sizeof(WsHeader) + align256((size_t)L * (size_t)F * 2);
}

int omni_shared_mlp_fwd(const omni_bf16 *x, const omni_bf16 *W_g, const omni_bf16 *W_u,
                        const omni_bf16 *W_d, int L, int d, int F, float *y, unsigned flags,
                        void *ws, size_t ws_bytes, omni_stream_t stream) {
    if (!x || !W_g || !W_u || !W_d || !y || !ws) return OMNI_ERR_INVALID_ARG;
    if (L <= 0 || d <= 0 || F <= 0 || (flags & ~OMNI_Y_ACCUMULATE) != 0)
        return OMNI_ERR_INVALID_ARG;
    if (d % 64 != 0 || F % 64 != 0) return OMNI_ERR_UNSUPPORTED;
    if ((int64_t)L * F > INT_MAX || (int64_t)L * d > INT_MAX || (int64_t)F * d > INT_MAX)
        return OMNI_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(W_g) || !aligned16(W_u) || !aligned16(W_d) || !aligned16(y))
        return OMNI_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return OMNI_ERR_INVALID_ARG;
    if (ws_bytes < omni_shared_mlp_workspace_size(L, d, F)) return OMNI_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    first_launch_in_call();
    if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), st) != cudaSuccess) return OMNI_ERR_CUDA;
    uint16_t *h = ws_at<uint16_t>(ws, sizeof(WsHeader));
    return cuda_rc(launch_shared_mlp(x, W_g, W_u, W_d, L, d, F, h, y,
                                     (flags & OMNI_Y_ACCUMULATE) != 0, ws_at<int>(ws, 0), st));
}

int omni_selftest_wait_timeout(void *ws, size_t ws_bytes, int limit_ms, omni_stream_t stream) {
    if (!ws || ws_bytes < sizeof(WsHeader) || limit_ms < 1 || limit_ms > 10000)
        return OMNI_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return OMNI_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), st) != cudaSuccess) return OMNI_ERR_CUDA;
    selftest_wait_kernel<<<1, 32, 0, st>>>(ws_at<int>(ws, 0), (uint64_t)limit_ms * 1000000ull);
    return cuda_rc(cudaGetLastError());
}

int omni_get_device_status(void *ws, size_t ws_bytes, omni_stream_t stream, int *status_out) {
    if (!ws || !status_out || ws_bytes < sizeof(WsHeader)) return OMNI_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int host = 0;
    if (cudaMemcpyAsync(&host, ws, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return OMNI_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return OMNI_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, sizeof(int), st) != cudaSuccess) return OMNI_ERR_CUDA;
    *status_out = host;
    return host == 0 ? OMNI_OK : OMNI_ERR_DEVICE;
}

}  // extern "C"

// omni_internal.h -- launchers shared between the .cu files of libomni and the
// workspace layout.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace omni {

constexpr int kSortTile = 2048;        // tasks per radix-sort tile

struct Sizes {
    int L, d, N_r, N_c, K, B;
    int64_t N, M, G;
    int Kr, Kc;          // row / column candidates: min(K, N_r), min(K, N_c)
    int C;               // merge candidates: cells (a, b) with (a+1)(b+1) <= K
    int64_t ntiles;      // radix tiles
    int qbits, passes;   // bits of the largest group id G - 1; radix passes of <= 8 bits
    // tensor-core path of the expert stage (expert_dense.cu)
    bool dense;          // laid out and run for this call
    int dense_thr;       // tasks that make an expert dense
    int dense_cap;       // dense columns at most (a multiple of 256)
};

struct WsLayout {
    size_t hdr, s_r, s_c, part_r, part_c, flags, row_val, row_idx, col_val, col_idx, idx, score, gate;
    size_t a_tok, a_exp, a_gate, b_tok, b_exp, b_gate, t_tok, t_exp, t_gate;
    size_t g_off, g_cnt, g_act, n_act, n_dist, bitmap, hist, tok_count, tok_slots;
    size_t dec_bar;          // grid-barrier word of the fused decode step (never cleared)
    size_t z_cnt, z_ndist;   // schedule counters (workspace copies)
    // tensor-core expert path: zeroed per call (dz_*), then the rest
    size_t dz_cnt, dz_ghot, dz_ccount;
    size_t d_ehot, d_list, d_whot, d_vt, d_G, d_P, d_ctok, d_cexp, d_cgate;
    size_t zero_end;         // [0, zero_end) must be zero when a call starts
    size_t total;
};

// Workspace regions.  Every call puts the 256-byte header at offset 0, then
// the counters of its regions that must start at zero (so one memset of
// [0, zero_end) clears them with the status word), then the rest of its
// regions in this order; the whole routed forward uses all of them, so
// omni_workspace_size (the full layout) covers every call.
enum WsRegion : unsigned {
    kRegRouter = 1u,      // s_r, s_c, axis candidates, idx / score / gate
    kRegSched = 2u,       // sort buffers, expert bitmap, radix histograms
    kRegSchedOut = 4u,    // sorted tasks and group arrays (routed forward only)
    kRegExpert = 8u,      // per-token slots of (expert, p) between the two expert kernels
    kRegDense = 16u,      // tensor-core expert path (only when Sizes::dense)
    kRegAll = 31u
};

bool make_sizes(int L, int d, int N_r, int N_c, int K, int B, Sizes *sz);
// Decides whether the tensor-core expert path runs for these sizes and flags
// (OMNI_EXPERT_DENSE / OMNI_EXPERT_SPARSE force it on / off) and sets its
// threshold and column cap.
void set_dense(Sizes *sz, unsigned flags);
WsLayout make_layout(const Sizes &sz, unsigned regions);
int merge_candidates(int K, int Kr, int Kc);

template <typename T>
inline T *ws_at(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

// ---- router GEMM (tcgen05): s_r = x W_r^T, s_c = x W_c^T (fp32)
// part_r [L, 2 * ceil(N_r/224)] and part_c: per (token, tile, column half) the max
// of s and the sum of exp(s - max), as float pairs ((-inf, 0) if empty).
cudaError_t launch_router_gemm(const uint16_t *x, const uint16_t *W_r, const uint16_t *W_c,
                               int L, int d, int N_r, int N_c, float *s_r, float *s_c,
                               float *part_r, float *part_c, int *status, cudaStream_t st);
constexpr int kGemmPartCols = 112;         // columns per LogSoftmax partial (two per 224-column tile)

// ---- router projection for a handful of tokens (no LogSoftmax partials)
bool router_small_ok(int L, int d);
cudaError_t launch_router_small(const uint16_t *x, const uint16_t *W_r, const uint16_t *W_c,
                                int L, int d, int N_r, int N_c, float *s_r, float *s_c,
                                cudaStream_t st);

// ---- per-axis LogSoftmax (optional) + top-K; then grid merge + gates
// With part_r / part_c (from the router GEMM) the LogSoftmax uses the
// per-tile partials; without them it computes max and sum itself.
cudaError_t launch_axis_topk(const float *in_r, const float *in_c, bool logsoftmax,
                             const float *part_r, const float *part_c,
                             float *p_r_out, float *p_c_out, int L, int N_r, int N_c, int K,
                             float *row_val, int *row_idx, float *col_val, int *col_idx,
                             int *flags, int *status, cudaStream_t st);
// dead_r / dead_c: the router GEMM's logits in the workspace, dropped from
// L2 once read (null: nothing is dropped, e.g. caller-owned log-probabilities)
// prep (may be null): run the schedule's per-token step (sched_token.cuh)
// on the merged selection too
struct SchedPrep;
cudaError_t launch_merge_topk(const float *row_val, const int *row_idx, const float *col_val,
                              const int *col_idx, int L, int N_c, int K, int Kr, int Kc, int C,
                              int32_t *idx, float *score, float *gate, const float *dead_r,
                              const float *dead_c, int N_r, const SchedPrep *prep,
                              cudaStream_t st);

// ---- fused decode step (L <= 16, K <= 128, d % 256 == 0, d <= 2048): the
// router projection, the selection and the token-order expert work in one
// cooperative launch; `bar` (one word) must be zero when it starts.
bool decode_fused_ok(int L, int d, int N_r, int N_c, int K, int Kr, int Kc, int C);
cudaError_t launch_decode_fused(const uint16_t *x, const uint16_t *W, const uint16_t *V,
                                const uint16_t *W_r, const uint16_t *W_c, int L, int d, int N_r,
                                int N_c, int K, int Kr, int Kc, int C, float *s_r, float *s_c,
                                float *row_val, int *row_idx, float *col_val, int *col_idx,
                                int32_t *idx, float *score, float *gate, float *y,
                                bool accumulate, unsigned long long *bar, unsigned epoch,
                                int *status, cudaStream_t st);

// ---- the pages' blockwise grid top-K (alternative to axis + merge); its
// candidates need L * blockwise_bands(...) * K * 16 bytes at `cand`
int blockwise_bands(int N_r, int N_c, int K);
cudaError_t launch_topk_blockwise(const float *p_r, const float *p_c, int L, int N_r, int N_c,
                                  int K, void *cand, int32_t *idx, float *score, float *gate,
                                  cudaStream_t st);

// ---- schedule (expects [0, lay.zero_end) of ws zeroed)
cudaError_t launch_schedule(const int32_t *idx, const float *gate, const Sizes &sz,
                            int32_t *task_token, int32_t *task_expert, float *task_gate,
                            int32_t *group_offsets, int32_t *group_counts,
                            int32_t *active_groups, int32_t *num_active, int32_t *num_distinct,
                            void *ws, const WsLayout &lay, cudaStream_t st, bool prepared = false,
                            bool any_order = false);
int sched_pass_width(const Sizes &sz);
uint32_t sched_pass_mask(const Sizes &sz, int p);
SchedPrep sched_prep_of(const Sizes &sz, void *ws, const WsLayout &lay);
// the radix scatter combines equal histogram increments of a warp (crowded
// groups, see schedule.cu)
bool sched_aggregate(const Sizes &sz);
// with any_order, launch_schedule groups the tasks by q without ordering a
// group's tasks by (token, expert) (one scan and one scatter instead of the
// radix passes); the per-token step then need not count the first pass's
// digits nor sort a token's experts
bool sched_unordered(const Sizes &sz);

// ---- grouped expert stage (expects the per-token slot counters zeroed).
// task_token == nullptr: the tasks are in token order, task m belongs to
// token m / K (task_expert / task_gate are then the router's idx / gate).
// group_offsets (nullable): each task is checked to lie in its group's range.
// dyn_M (nullable): the number of tasks is read from the device (the
// compacted list of the tensor-core path), M is then an upper bound.
cudaError_t launch_grouped_expert(const uint16_t *x, const uint16_t *W, const uint16_t *V,
                                  const Sizes &sz, const int32_t *task_token,
                                  const int32_t *task_expert, const float *task_gate,
                                  float *y, bool accumulate, void *ws, const WsLayout &lay,
                                  cudaStream_t st, const int32_t *group_offsets = nullptr,
                                  const int32_t *dyn_M = nullptr);

// ---- tensor-core expert path (expert_dense.cu); expects the dz_* regions
// zeroed.  prepare: dense experts per active group, their columns, W_D and
// V_D^T, G (gates of their tasks) and the compacted list of the other tasks;
// gemms: P = G . SiLU(x W_D^T), then y += P V_D.
struct DenseWs {
    int32_t *cnt;            // [N] tasks per expert, then -(column + 1) for dense ones
    int32_t *ghot;           // [G + 1] dense experts per group, then their first column
    int32_t *ehot;           // [1] dense experts found (before the cap)
    int32_t *ccount;         // [2] compacted tasks; tasks covered by the active groups
    int32_t *list;           // [cap] dense expert ids by column
    uint16_t *whot, *vt;     // [cap, d], [d, cap] bf16
    float *G;                // [L, cap]
    uint16_t *P;             // [L, cap] bf16
    int32_t *c_tok, *c_exp;  // [M] compacted tasks
    float *c_gate;
    int cap, thr;
};
DenseWs dense_ws_of(const Sizes &sz, void *ws, const WsLayout &lay);
cudaError_t launch_dense_prepare(const uint16_t *W, const uint16_t *V, const Sizes &sz,
                                 const int32_t *task_token, const int32_t *task_expert,
                                 const float *task_gate, const int32_t *group_offsets,
                                 const int32_t *active_groups, const int32_t *num_active,
                                 const DenseWs &o, int *status, cudaStream_t st);
cudaError_t launch_dense_gemms(const uint16_t *x, const Sizes &sz, const DenseWs &o, float *y,
                               int *status, cudaStream_t st);
// exclusive scan of n ints in place (one CTA); the total goes to *total
cudaError_t launch_exclusive_scan(int32_t *a, int64_t n, int32_t *total, cudaStream_t st);

// ---- backward of the routed branch (selection fixed)
cudaError_t launch_routed_bwd(const uint16_t *x, const uint16_t *W, const uint16_t *V,
                              const uint16_t *W_r, const uint16_t *W_c, const Sizes &sz,
                              const int32_t *idx, const float *gate, const float *dy, float *dx,
                              float *dW, float *dV, float *dW_r, float *dW_c, uint32_t *seen,
                              uint32_t *shared_rows, int *rcnt, int2 *rslots, int rcap,
                              int *status, cudaStream_t st);
// slots per router row in the backward's lists (a row used by more tokens
// reduces the extra pairs into dW_r / dW_c directly)
constexpr int kBwdRowCap = 256;

// ---- shared dense MLP (two tile GEMMs; h is [L, F] bf16 scratch)
cudaError_t launch_shared_mlp(const uint16_t *x, const uint16_t *W_g, const uint16_t *W_u,
                              const uint16_t *W_d, int L, int d, int F, uint16_t *h, float *y,
                              bool accumulate, int *status, cudaStream_t st);

int device_sm_count();

}  // namespace omni

/*
 * omni.h -- C ABI of the B200 (sm_100a) routed-branch forward of an OmniMoE
 * layer (with its backward, and the shared dense MLP the layer adds to it).
 * Library: atomic_expert_layer_b200/libomni.so.
 *
 * Sources, cited by page title and section:
 *   [R] "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale",
 *       review at paper.rainbus.top, method paragraph (steps 1-3: atomic
 *       experts and Dynamic Expert Assembly; Cartesian product router;
 *       expert-centric scheduling with grouped GEMM).
 *   [G] same title, gist.science summary, section 2.1 (atomic experts, DEA,
 *       shared MLP) and section 2.2 (Cartesian product router; expert-centric
 *       scheduling: task collection, grouping by contiguous expert-id ranges,
 *       token order inside a group, grouped GEMM).
 *
 * Notation follows [R]: L tokens of width d; N = N_r * N_c atomic experts,
 * expert n sits at grid cell (i, j) with n = i * N_c + j; W and V hold the
 * w_in and w_out vectors of all experts as rows (N x d); W_r, W_c are the
 * router projections; K experts are selected per token; B experts form a
 * group, expert e belongs to group q = e / B; G = ceil(N / B) groups;
 * M = L * K tasks.
 *
 * Conventions shared by every entry point:
 *   - All array arguments are DEVICE pointers to caller-owned, contiguous,
 *     row-major buffers.  The library never allocates or frees device memory;
 *     scratch comes from the caller's workspace `ws` of `ws_bytes` bytes, at
 *     least omni_workspace_size(...) for the same sizes (or the size function
 *     named at the call), 256-byte aligned.
 *     One workspace must not be used by two calls that overlap in time.
 *   - bf16 values are passed as their 16-bit patterns (omni_bf16).
 *   - W_r is stored as N_r rows of d (row i is the routing vector of grid row
 *     i), i.e. the d x N_r matrix of [R] in column-major order; likewise W_c.
 *     Then s_r = x W_r^T in this storage.
 *   - Every call enqueues its work on `stream` (NULL = legacy default stream)
 *     and returns without synchronising.  Pointers must stay valid until the
 *     stream reaches the work.
 *   - Return value: OMNI_OK, or a negative omni_status.  Argument problems are
 *     found on the host before anything is enqueued.  OMNI_ERR_CUDA means a
 *     launch failed.  Problems found on the device (an expert id out of range,
 *     a bounded wait that ran out) are recorded in a status word inside `ws`;
 *     read it with omni_get_device_status.  Each entry point clears that word
 *     when it starts.  No function prints, throws or exits.
 *   - bf16 pointers must be 16-byte aligned; d must be a multiple of 8.
 */
#ifndef OMNI_H_
#define OMNI_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                 /* = cudaStream_t */
typedef struct CUstream_st *omni_stream_t;
typedef uint16_t omni_bf16;         /* bf16 bit pattern */

typedef enum {
    OMNI_OK = 0,
    OMNI_ERR_INVALID_ARG = -1,      /* null pointer, non-positive size, K > N, misaligned pointer */
    OMNI_ERR_UNSUPPORTED = -2,      /* a size outside what the kernels handle (see each call)    */
    OMNI_ERR_WORKSPACE = -3,        /* ws_bytes below omni_workspace_size(...)                    */
    OMNI_ERR_CUDA = -4,             /* a CUDA launch or runtime call failed                      */
    OMNI_ERR_DEVICE = -5            /* recorded on the device; see omni_get_device_status        */
} omni_status;

/* flags */
#define OMNI_ROUTER_LOGPROBS_IN 1u  /* omni_router_topk: p_r, p_c are inputs (skip s = xW^T and LogSoftmax) */
#define OMNI_Y_ACCUMULATE       2u  /* y += routed(x) instead of y = routed(x)                           */
#define OMNI_TOKEN_ORDER        4u  /* omni_routed_fwd: expert stage in token order, no schedule (below)  */
#define OMNI_TOPK_BLOCKWISE     8u  /* omni_router_topk: the pages' blockwise grid top-K (below)           */
#define OMNI_EXPERT_DENSE      16u  /* expert stage: always try the tensor-core tiles for dense experts   */
#define OMNI_EXPERT_SPARSE     32u  /* expert stage: every task on the task-by-task path (no tiles)       */

/* Device status codes written into the workspace status word. */
#define OMNI_DEV_OK              0
#define OMNI_DEV_BAD_EXPERT      1  /* an expert id outside [0, N) reached the schedule   */
#define OMNI_DEV_WAIT_TIMEOUT    2  /* a bounded barrier wait ran out (no hang)           */
#define OMNI_DEV_BAD_SCHEDULE    3  /* schedule arrays inconsistent (offsets/ids)          */

/* Size limits of the library (OMNI_ERR_UNSUPPORTED beyond them). */
#define OMNI_MAX_AXIS   8192        /* N_r, N_c                                   */
#define OMNI_MAX_K      512         /* K                                          */
#define OMNI_MAX_B      1024        /* B                                          */
#define OMNI_MAX_D      2048        /* d for the expert stage; d % 256 == 0 there */

/* Library version, for the binding's sanity check. */
int omni_version(void);

/* Human-readable name of an omni_status or a device status code (static string). */
const char *omni_status_string(int status);
const char *omni_device_status_string(int dev_status);

/*
 * Bytes of workspace that every entry point needs for these sizes (the same
 * layout serves all four calls) with flags 0.  Returns 0 if the sizes are
 * invalid.
 */
size_t omni_workspace_size(int L, int d, int N_r, int N_c, int K, int B);

/*
 * The same for calls made with `flags`: OMNI_EXPERT_DENSE needs room for
 * the tensor-core expert path at any size, OMNI_EXPERT_SPARSE none, and
 * OMNI_TOKEN_ORDER (omni_routed_fwd only) leaves out the schedule and the
 * tensor-core path.  omni_workspace_size(...) is this with flags 0.
 */
size_t omni_workspace_size_flags(int L, int d, int N_r, int N_c, int K, int B, unsigned flags);

/* Smaller workspaces for the three stage calls used on their own (each is at
 * most omni_workspace_size of the same sizes).  0 for invalid sizes. */
size_t omni_router_workspace_size(int L, int N_r, int N_c, int K);
size_t omni_schedule_workspace_size(int L, int K, int N, int B);
size_t omni_expert_workspace_size(int L, int d, int K, int N, int B);
/* omni_grouped_expert_fwd called with `flags` (OMNI_EXPERT_DENSE needs more). */
size_t omni_expert_workspace_size_flags(int L, int d, int K, int N, int B, unsigned flags);

/*
 * Cartesian product router, [R] step 2 and [G] section 2.2.
 *   s_r = x W_r^T, s_c = x W_c^T            (bf16 inputs, fp32 accumulation)
 *   p_r = LogSoftmax(s_r), p_c = LogSoftmax(s_c)   (fp32, per token)
 *   S_ij = p_r[i] + p_c[j]  (one fp32 addition; the N-entry grid is never built)
 * and the exact global top-K of S per token, ordered by the key
 *   (S desc, p_r[i] desc, p_c[j] desc, n asc),
 * with gates g = softmax of the K selected S (the pages leave g_x open; this
 * is the reading taken).
 *   x    [L, d]   bf16          W_r [N_r, d] bf16      W_c [N_c, d] bf16
 *   p_r  [L, N_r] fp32  output, or input with OMNI_ROUTER_LOGPROBS_IN
 *   p_c  [L, N_c] fp32  output, or input with OMNI_ROUTER_LOGPROBS_IN
 *   idx  [L, K]   int32 output, n = i * N_c + j, in key order
 *   score[L, K]   fp32  output, S of each selected cell
 *   gate [L, K]   fp32  output, softmax over the token's K scores
 * With OMNI_ROUTER_LOGPROBS_IN, x / W_r / W_c / d are not read (may be NULL / 0).
 * Row and column candidates are the top min(K, N_r) rows and min(K, N_c)
 * columns.  Limits: K <= N_r * N_c, K <= OMNI_MAX_K, N_r, N_c <= OMNI_MAX_AXIS.
 * p must be finite (NaN / Inf give an unspecified but in-range selection).
 * OMNI_TOPK_BLOCKWISE (with OMNI_ROUTER_LOGPROBS_IN only): the same result by
 * the selection [R] step 2 describes -- the implicit grid cut into blocks of
 * rows, each scored cell by cell by a thread block that keeps its local
 * top-K, then a per-token merge -- instead of the row / column pruning.  It
 * scores all N_r * N_c cells (an alternative kept for comparison).  Extra
 * limit: K <= (N_r + N_c) / 4, else OMNI_ERR_UNSUPPORTED.
 */
int omni_router_topk(const omni_bf16 *x, const omni_bf16 *W_r, const omni_bf16 *W_c,
                     int L, int d, int N_r, int N_c, int K,
                     float *p_r, float *p_c, int32_t *idx, float *score, float *gate,
                     unsigned flags, void *ws, size_t ws_bytes, omni_stream_t stream);

/*
 * Expert-centric scheduling, [R] step 3 and [G] section 2.2.
 * Task m = t * K + k is (token t, expert e = idx[t, k], gate[t, k]).  Tasks are
 * sorted by (q = e / B, t, e) -- group id, then token id, then expert id (the
 * pages fix the first two keys; the third makes the order unique) -- and the
 * groups are bucketed:
 *   task_token, task_expert [M] int32, task_gate [M] fp32   sorted tasks
 *   group_offsets [G + 1] int32   exclusive prefix sum of group_counts
 *   group_counts  [G]     int32   tasks per group
 *   active_groups [G]     int32   groups with >= 1 task, ascending; entries
 *                                 past num_active are left unspecified
 *   num_active    [1]     int32   number of active groups
 *   num_distinct  [1]     int32   number of distinct experts among the tasks
 * idx [L, K] int32 and gate [L, K] fp32 are inputs (e.g. from omni_router_topk);
 * expert ids must lie in [0, N) and be distinct within a token.  An id out of
 * range sets OMNI_DEV_BAD_EXPERT; that task is then given expert 0 and gate 0
 * so that every later access stays in bounds.
 * Limits: M <= 2^31 - 1, B <= OMNI_MAX_B, K <= OMNI_MAX_K.
 * The output is bit-identical from run to run (the sort key is unique).
 */
int omni_schedule(const int32_t *idx, const float *gate, int L, int K, int N, int B,
                  int32_t *task_token, int32_t *task_expert, float *task_gate,
                  int32_t *group_offsets, int32_t *group_counts, int32_t *active_groups,
                  int32_t *num_active, int32_t *num_distinct,
                  void *ws, size_t ws_bytes, omni_stream_t stream);

/*
 * Grouped expert computation, [R] steps 1 and 3 and [G] section 2.2
 * ("grouped GEMM"): for every active group q with tokens X_q, expert rows
 * W_q, V_q and gate matrix G_q (gate of task (t, e), 0 where there is none),
 *   O_q = (G_q . SiLU(X_q W_q^T)) V_q,      y[t] += O_q[t]  for its tokens.
 * sigma is read as SiLU (one w_in per expert leaves SwiGLU without a gate).
 *   x [L, d] bf16, W [N, d] bf16, V [N, d] bf16
 *   schedule arrays as produced by omni_schedule for the same L, K, N, B
 *   y [L, d] fp32  output (overwritten, or accumulated with OMNI_Y_ACCUMULATE)
 * Two execution paths share the work, by how dense G_q is:
 *   - tensor cores, for the "dense" experts: those that at least
 *     thr = max(32, ceil(L / 96)) tasks use.  The active groups are walked
 *     (active_groups, num_active, group_offsets); every group's dense experts
 *     become columns of one bf16 tile GEMM over all L tokens,
 *       P = G . SiLU(x W_D^T)  (P rounded to bf16),   y += P V_D,
 *     with G the gates of their tasks (0 elsewhere).  At most a few thousand
 *     columns are built (a cap set by L); the experts past it stay on the
 *     other path.
 *   - CUDA cores, task by task, for every other task: P = g SiLU(x_t . w_e)
 *     for the task pairs only (fp32), then y_t = sum of p V[e] per token.
 *   By default the tensor-core path is tried when L * K * d >= 2^31 (large
 *   stages; below that an expert rarely reaches thr and its fixed cost is
 *   not paid).  OMNI_EXPERT_DENSE tries it at any size (the workspace must
 *   then come from omni_workspace_size_flags with that flag);
 *   OMNI_EXPERT_SPARSE never does.  When no expert is dense the tiles do no
 *   work.
 * Checks on the device (OMNI_DEV_BAD_SCHEDULE): every task must lie in its
 * group's range of group_offsets; on the tensor-core path also num_active in
 * [0, G], active group ids in range, offsets non-decreasing within [0, M],
 * each group's tasks of its own experts, and the active groups covering all
 * L * K tasks.
 * Each y row gets the CUDA-core sum in the order slots were claimed (atomic
 * counters) and the tile sum in a fixed order, so y may differ in the last
 * bits between runs.  Limits: d % 256 == 0, d <= OMNI_MAX_D, B <= OMNI_MAX_B.
 */
int omni_grouped_expert_fwd(const omni_bf16 *x, const omni_bf16 *W, const omni_bf16 *V,
                            int L, int d, int K, int N, int B,
                            const int32_t *task_token, const int32_t *task_expert,
                            const float *task_gate, const int32_t *group_offsets,
                            const int32_t *active_groups, const int32_t *num_active,
                            float *y, unsigned flags, void *ws, size_t ws_bytes,
                            omni_stream_t stream);

/*
 * The whole routed branch: omni_router_topk, the schedule and
 * omni_grouped_expert_fwd back to back on `stream`, with every intermediate in
 * `ws` and no host synchronisation:  y = routed(x)  (the shared dense MLP of
 * [G] section 2.1 is not part of it).  OMNI_EXPERT_DENSE / OMNI_EXPERT_SPARSE
 * choose the expert stage's paths as for omni_grouped_expert_fwd (its
 * schedule is produced here, so its offsets are not re-checked).  The
 * schedule built here only groups the tasks by q = e / B, with no order
 * inside a group (the expert stage needs no more; omni_schedule returns the
 * full (group, token, expert) order).
 *   x [L, d], W [N, d], V [N, d], W_r [N_r, d], W_c [N_c, d]  bf16
 *   y [L, d] fp32 output;  idx_out [L, K] int32, gate_out [L, K] fp32 are
 *   optional copies of the routing (NULL to skip).
 * Token order: with flag OMNI_TOKEN_ORDER, and always for L <= 16 tokens,
 * the expert stage takes the tasks in token order straight from the router
 * (task t*K + k = (t, idx[t,k], gate[t,k])) and the schedule is skipped.
 * For L <= 16 (d <= 2048, K <= 128, within the kernel's shared memory) the
 * whole step is one cooperative launch (projection, per-token selection and
 * gates, expert work, separated by bounded grid barriers); it clears its own
 * status word and needs no cleared workspace.
 * y is the same sum (up to summation order); only the order in which expert
 * rows are fetched changes.  For a few tokens the grouping has nothing to
 * reuse and the schedule's launches are pure latency; for large batches the
 * flag is the token-centric execution the expert-centric schedule replaces
 * (an ablation); it needs only omni_workspace_size_flags(..., OMNI_TOKEN_ORDER)
 * bytes and never uses the tensor-core path.
 * Limits: those of the three calls above.
 */
int omni_routed_fwd(const omni_bf16 *x, const omni_bf16 *W, const omni_bf16 *V,
                    const omni_bf16 *W_r, const omni_bf16 *W_c,
                    int L, int d, int N_r, int N_c, int K, int B,
                    float *y, int32_t *idx_out, float *gate_out,
                    unsigned flags, void *ws, size_t ws_bytes, omni_stream_t stream);

/*
 * Backward of the routed branch.  The pages give the forward only; this is
 * its derivative with the forward's top-K selection held fixed (a selection
 * has no gradient).  Per task (t, k), e = idx[t,k], g = gate[t,k]:
 *   h = x_t . w_e, a = SiLU(h), c = dy_t . v_e,  dgate = a c,
 *   dV[e] += g a dy_t,  dW[e] += g c SiLU'(h) x_t,  dx_t += g c SiLU'(h) w_e;
 * through the gate softmax dS_k = g_k (dgate_k - sum_j g_j dgate_j), through
 * S = p_r[i] + p_c[j] and the LogSoftmax (whose dense term vanishes because
 * the selected gates sum to 1) the router gradient is sparse:
 *   dx_t += dS_k (W_r[i] + W_c[j]),  dW_r[i] += dS_k x_t,  dW_c[j] += dS_k x_t.
 *   x [L, d], W, V [N, d], W_r [N_r, d], W_c [N_c, d]  bf16 (the forward's)
 *   idx [L, K] int32, gate [L, K] fp32  the forward's routing (omni_router_topk,
 *                                       or omni_routed_fwd's idx_out / gate_out)
 *   dy [L, d] fp32     gradient of the loss with respect to y
 *   dx [L, d] fp32     output, overwritten
 *   dW, dV [N, d] fp32 accumulated (+=) in the rows of the experts used
 *   dW_r [N_r, d], dW_c [N_c, d] fp32  accumulated (+=)
 * ws: at least 256 bytes (the status word).  With at least
 * omni_routed_bwd_workspace_size() bytes the call first marks, in two
 * bitmaps over the N experts, the experts that more than one task uses; the
 * dW and dV rows of every other expert then get one plain read-add-write
 * (the fastest path, and bit-reproducible), and only the shared rows go
 * through fp32 reductions, whose last bits vary between runs.  The router
 * rows' dW_r / dW_c then collect their tokens' (token, dS) pairs in lists of
 * up to 256 per row, summed by a second kernel (one plain read-add-write per
 * row; a row with more pairs reduces the extra ones directly).  With room
 * for the bitmaps only, the router rows are reduced; with 256 bytes, every
 * row is.  All fp32 arrays 16-byte aligned.
 * Limits: d % 256 == 0, d <= OMNI_MAX_D, K <= OMNI_MAX_K.
 */
int omni_routed_bwd(const omni_bf16 *x, const omni_bf16 *W, const omni_bf16 *V,
                    const omni_bf16 *W_r, const omni_bf16 *W_c,
                    int L, int d, int N_r, int N_c, int K,
                    const int32_t *idx, const float *gate, const float *dy,
                    float *dx, float *dW, float *dV, float *dW_r, float *dW_c,
                    unsigned flags, void *ws, size_t ws_bytes, omni_stream_t stream);

/* Workspace bytes of omni_routed_bwd with its expert bitmaps and router-row
 * lists: 256, two bitmaps of N bits (each rounded up to 256 bytes), a counter
 * per router row (N_r + N_c int32, rounded up to 256 bytes) and 256 slots of
 * 8 bytes per router row (0 for invalid sizes).  The pages have no
 * counterpart; it only sizes the backward's scratch. */
size_t omni_routed_bwd_workspace_size(int L, int d, int N_r, int N_c, int K);

/*
 * The shared dense MLP that the layer adds to the routed branch
 * ("OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale",
 * rainbus review page, method paragraph, step 1: y = routed(x) + MLP(x);
 * gist.science summary (German edition), section 2.1 "Kernkomponenten": a
 * standard dense MLP branch, active for every input).  The pages give no
 * form; this is the gated one with hidden width F:
 *   h = SiLU(x W_g^T) * (x W_u^T)      [L, F], held in bf16 in ws
 *   y = h W_d^T,  or  y += h W_d^T with OMNI_Y_ACCUMULATE
 * so omni_routed_fwd followed by this call with OMNI_Y_ACCUMULATE gives the
 * whole layer's output.
 *   x [L, d] bf16;  W_g, W_u [F, d] bf16 (one row per hidden unit);
 *   W_d [d, F] bf16 (one row per output feature);  y [L, d] fp32.
 * Products run on the tensor cores (bf16 in, fp32 accumulate); each y element
 * is written by one tile, so the result is the same on every run.
 * ws: omni_shared_mlp_workspace_size(L, d, F) bytes, 256-byte aligned.  All
 * arrays 16-byte aligned.  flags: 0 or OMNI_Y_ACCUMULATE.
 * Limits: d % 64 == 0, F % 64 == 0, L * F, L * d and F * d < 2^31
 * (OMNI_ERR_UNSUPPORTED beyond).
 */
size_t omni_shared_mlp_workspace_size(int L, int d, int F);
int omni_shared_mlp_fwd(const omni_bf16 *x, const omni_bf16 *W_g, const omni_bf16 *W_u,
                        const omni_bf16 *W_d, int L, int d, int F, float *y, unsigned flags,
                        void *ws, size_t ws_bytes, omni_stream_t stream);

/*
 * omni_grouped_expert_fwd without a workspace, for callers that cannot
 * allocate device memory when they run the layer (a serving runtime whose
 * memory is planned once at start-up, code where cudaMalloc is not allowed).
 * The pages have no counterpart; it is a deployment convenience.
 * Same arguments and result as omni_grouped_expert_fwd, minus ws / ws_bytes.
 * Its scratch is a fixed array inside the library (about 2 MB on every GPU
 * that loads it, held until the process exits), so:
 *   - sizes are limited to L <= 16384 tokens and L * K <= 262144 tasks
 *     (OMNI_ERR_UNSUPPORTED beyond), besides the limits of the workspace call;
 *   - every call on a device shares the array: calls that overlap on the GPU
 *     (different streams, or different host threads) race and must not be
 *     issued; the array keeps the last call's contents, and the call clears
 *     what has to start at zero itself;
 *   - the array's device address is looked up (cudaGetSymbolAddress) on the
 *     first call made in each CUDA context, with that context current, and
 *     kept for later calls in the same context; make that first call before
 *     capturing a stream into a CUDA graph.  A context created later for the
 *     same device (after cudaDeviceReset, or a driver-API context other than
 *     the primary one) gets its own lookup on its first call;
 *   - device-detected problems are recorded in the array's own status word,
 *     which omni_get_device_status cannot read: read it with
 *     omni_noalloc_get_device_status.
 * No device memory is allocated or freed.
 */
int omni_grouped_expert_fwd_noalloc(const omni_bf16 *x, const omni_bf16 *W, const omni_bf16 *V,
                                    int L, int d, int K, int N, int B,
                                    const int32_t *task_token, const int32_t *task_expert,
                                    const float *task_gate, const int32_t *group_offsets,
                                    const int32_t *active_groups, const int32_t *num_active,
                                    float *y, unsigned flags, omni_stream_t stream);

/*
 * The status word of omni_grouped_expert_fwd_noalloc's array on the current
 * device: synchronises `stream`, copies the word into *status_out (an
 * OMNI_DEV_* code, e.g. OMNI_DEV_BAD_SCHEDULE for a task whose expert or
 * token id is out of range) and clears it.  Allocates nothing.  Returns
 * OMNI_ERR_DEVICE when the word was set, OMNI_OK when it was clear.
 */
int omni_noalloc_get_device_status(omni_stream_t stream, int *status_out);

/*
 * Diagnostic, not part of the layer: launches one CTA that waits on a
 * shared-memory barrier nothing ever arrives at, through the same bounded
 * wait the pipelined kernels use, with its limit set to `limit_ms`
 * (1..10000).  The wait runs out, the kernel records OMNI_DEV_WAIT_TIMEOUT in
 * the status word of `ws` and returns; the context stays usable.  Tests use
 * it to check that a stuck wait ends with a status, not a hang.
 */
int omni_selftest_wait_timeout(void *ws, size_t ws_bytes, int limit_ms, omni_stream_t stream);

/*
 * Synchronises `stream`, copies the status word of `ws` into *status_out
 * (an OMNI_DEV_* code) and clears it.  For tests and error handling; it is
 * the only call that blocks the host.
 */
int omni_get_device_status(void *ws, size_t ws_bytes, omni_stream_t stream, int *status_out);

#ifdef __cplusplus
}
#endif

#endif /* OMNI_H_ */

// schedule.cu -- expert-centric scheduling on sm_100a.
//
// "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale"
// (rainbus review page, method paragraph, step 3; gist.science summary,
// section 2.2 "Experten-zentriertes Scheduling"): the L*K routing decisions
// are flattened into tasks (token, expert, gate), sorted by expert id,
// bucketed into groups of B consecutive expert ids and ordered inside a
// group by token id.  The order used here is (q = e / B, t, e): unique per
// task, so the result does not depend on the sort's internals.
//
// Pipeline (no host synchronisation, no spin-waits):
//   1. prepare (warp per token): sort the token's K tasks by expert id, write
//      them in (t, e) order, count tasks per group, count distinct experts
//      (the first task to set an expert's bit in a bitmap counts it), and
//      count the first radix pass's digits per 2048-task tile (atomics).
//   2. scans (one launch, two CTAs): group offsets and active-group list;
//      the first pass's digit-major histogram.
//   3. LSD radix sort of the tasks on q alone, digits of <= 8 bits, stable.
//      The input is in (t, e) order, so a stable sort by q yields (q, t, e).
//      Each pass: stable scatter (warps rank equal digits with
//      __match_any_sync, in input order) that also counts the next pass's
//      digits of its output, then one scan of that histogram.
#include "omni_common.cuh"
#include "omni_internal.h"
#include "sched_token.cuh"

namespace omni {
namespace {

constexpr int kScatterThreads = 256;                       // 8 warps
constexpr int kItemsPerWarp = kSortTile / (kScatterThreads / 32);   // 256

// ------------------------------------------------------------ radix digits
__device__ __forceinline__ uint32_t digit_of(int32_t e, int B, int shift, uint32_t dmask) {
    return sched_digit(e, B, shift, dmask);
}

// ---------------------------------------------------------- 1. prepare
// Warp per token: sort the token's K tasks by expert id, write them at
// t*K + rank, count tasks per group, mark experts, and count the first radix
// pass's digits per tile (so no separate histogram pass is needed).
__global__ void sched_prepare_kernel(const int32_t *__restrict__ idx,
                                     const float *__restrict__ gate, int L, int K, int N, int B,
                                     int32_t *__restrict__ a_tok, int32_t *__restrict__ a_exp,
                                     float *__restrict__ a_gate, int32_t *__restrict__ counts,
                                     uint32_t *__restrict__ bitmap, int32_t *__restrict__ num_distinct,
                                     int32_t *__restrict__ hist0, int64_t ntiles, uint32_t dmask0,
                                     int *status) {
    extern __shared__ int32_t sh_e[];
    grid_dependency_wait();
    grid_dependents_launch();
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    const int t = blockIdx.x * (blockDim.x >> 5) + warp;
    if (t >= L) return;
    int32_t *e_s = sh_e + (size_t)warp * K;
    const size_t row = (size_t)t * K;
    for (int k = lane; k < K; k += 32) {
        int32_t e = idx[row + k];
        if (e < 0 || e >= N) {
            set_status(status, OMNI_DEV_BAD_EXPERT);
            e = 0;                                         // keep every access in range
        }
        e_s[k] = e;
    }
    __syncwarp();
    SchedPrep o;
    o.a_tok = a_tok; o.a_exp = a_exp; o.a_gate = a_gate;
    o.counts = counts; o.bitmap = bitmap; o.num_distinct = num_distinct;
    o.hist0 = hist0; o.ntiles = ntiles; o.dmask0 = dmask0; o.B = B; o.unordered = 0;
    sched_token(o, t, K, e_s, [&](int u) {
        const int32_t raw = idx[row + u];
        return (raw < 0 || raw >= N) ? 0.f : gate[row + u];
    });
}

// ------------------------------------------------ block scan (1024 threads)
// Exclusive scan of one int per thread; returns the block total in *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int *sh32, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int incl = warp_iscan(v);
    __syncthreads();                       // sh32 may still be read by a previous call
    if (lane == 31) sh32[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int s = sh32[lane];
        const int is = warp_iscan(s);
        sh32[lane] = is - s;
        if (lane == 31) sh32[32] = is;
    }
    __syncthreads();
    *total = sh32[32];
    return sh32[warp] + incl - v;
}

constexpr int kScanTile = 4096;            // elements per tile: 1024 threads x 4

// In-place exclusive scan of a[0..n) by one CTA of 1024 threads.  Tiles of
// 4096 are loaded coalesced (the next tile's loads are issued before the
// current tile is scanned) and staged through shared memory so each thread
// owns 4 consecutive elements.  If `tail` is non-null the total is written
// there.
constexpr int kFastPer = 16;                               // elements per thread
constexpr int64_t kFastScan = 1024 * kFastPer;             // one-shot scan limit

// One-shot scan of n <= kFastScan ints by 1024 threads.  Warp w owns the
// contiguous chunk [512 w, 512 w + 512); lane l holds its elements
// 32 k + l (k < 16), so every load and store is a coalesced 128-byte row.
// Loads the chunk into v, scans the warp totals across the CTA and returns
// the exclusive prefix of the warp's first element; *total is the sum of all
// n.  With act_total, the count of positive elements is scanned the same way
// (*act_run0 = exclusive count before the warp, *act_total = all).
__device__ __forceinline__ int fast_load_scan(const int32_t *a, int64_t n, int *v, int *sh32,
                                              int *total, int *act_run0, int *act_total) {
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    const int64_t base = (int64_t)warp * (32 * kFastPer);
    int sum = 0, act = 0;
#pragma unroll
    for (int k = 0; k < kFastPer; ++k) {
        const int64_t i = base + k * 32 + lane;
        v[k] = i < n ? a[i] : 0;
        sum += v[k];
        act += v[k] > 0;
    }
    sum = warp_isum(sum);
    int run0 = block_exclusive_scan(lane == 0 ? sum : 0, sh32, total);
    run0 = __shfl_sync(0xffffffffu, run0, 0);
    if (act_total) {
        act = warp_isum(act);
        int ar = block_exclusive_scan(lane == 0 ? act : 0, sh32, act_total);
        *act_run0 = __shfl_sync(0xffffffffu, ar, 0);
    }
    return run0;
}

// Writes the exclusive scan of the chunk loaded by fast_load_scan.
__device__ __forceinline__ void fast_store_scan(int32_t *a, int64_t n, const int *v, int run) {
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    const int64_t base = (int64_t)warp * (32 * kFastPer);
#pragma unroll
    for (int k = 0; k < kFastPer; ++k) {
        const int incl = warp_iscan(v[k]);
        const int64_t i = base + k * 32 + lane;
        if (i < n) a[i] = run + incl - v[k];
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
}

__device__ void cta_exclusive_scan(int32_t *a, int64_t n, int32_t *tail, int *tile, int *sh32) {
    const int tid = threadIdx.x;
    if (n <= kFastScan) {
        int v[kFastPer];
        int total;
        const int run0 = fast_load_scan(a, n, v, sh32, &total, nullptr, nullptr);
        fast_store_scan(a, n, v, run0);
        if (tail && tid == 0) *tail = total;
        return;
    }
    int carry = 0;
    int nx[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int64_t i = (int64_t)k * 1024 + tid;
        nx[k] = i < n ? a[i] : 0;
    }
    for (int64_t base = 0; base < n; base += kScanTile) {
        __syncthreads();
#pragma unroll
        for (int k = 0; k < 4; ++k) tile[k * 1024 + tid] = nx[k];
        const int64_t nb = base + kScanTile;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int64_t i = nb + k * 1024 + tid;
            nx[k] = i < n ? a[i] : 0;
        }
        __syncthreads();
        int v[4], sum = 0;
        for (int k = 0; k < 4; ++k) {
            v[k] = tile[4 * tid + k];
            sum += v[k];
        }
        int total;
        int run = carry + block_exclusive_scan(sum, sh32, &total);
        for (int k = 0; k < 4; ++k) {
            tile[4 * tid + k] = run;
            run += v[k];
        }
        carry += total;
        __syncthreads();
        for (int k = 0; k < 4; ++k) {
            const int64_t i = base + k * 1024 + tid;
            if (i < n) a[i] = tile[k * 1024 + tid];
        }
    }
    if (tail && tid == 0) *tail = carry;
}

// ----------------------------------------------------- 2. group scan
// CTA 0: group offsets (exclusive scan of the counts), the caller's copy of
// the counts, active groups, the distinct-expert count.  CTA 1 (if a radix
// pass follows): exclusive scan of the first pass's digit-major histogram.
__global__ void __launch_bounds__(1024) sched_scan_kernel(
    const int32_t *__restrict__ counts, int64_t G, int32_t *__restrict__ counts_out,
    int32_t *__restrict__ offsets, int32_t *__restrict__ active, int32_t *__restrict__ num_active,
    const int32_t *__restrict__ ndist_acc, int32_t *__restrict__ num_distinct,
    int32_t *__restrict__ hist0, int64_t nhist) {
    __shared__ int tile[kScanTile];
    __shared__ int tile2[kScanTile];
    __shared__ int sh32[33];
    grid_dependency_wait();
    grid_dependents_launch();
    const int tid = threadIdx.x;
    if (blockIdx.x == 1) {
        cta_exclusive_scan(hist0, nhist, nullptr, tile, sh32);
        return;
    }
    if (tid == 0) *num_distinct = *ndist_acc;
    if (G <= kFastScan) {
        int v[kFastPer];
        int total, atotal, arun;
        int run = fast_load_scan(counts, G, v, sh32, &total, &arun, &atotal);
        const int warp = tid >> 5;
        const unsigned lane = lane_id();
        const int64_t base = (int64_t)warp * (32 * kFastPer);
#pragma unroll
        for (int k = 0; k < kFastPer; ++k) {
            const int incl = warp_iscan(v[k]);
            const unsigned act = __ballot_sync(0xffffffffu, v[k] > 0);
            const int64_t g = base + k * 32 + lane;
            if (g < G) {
                offsets[g] = run + incl - v[k];
                counts_out[g] = v[k];
                if (v[k] > 0) active[arun + __popc(act & lanemask_lt())] = (int32_t)g;
            }
            run += __shfl_sync(0xffffffffu, incl, 31);
            arun += __popc(act);
        }
        if (tid == 0) {
            offsets[G] = total;
            *num_active = atotal;
        }
        return;
    }
    int carry = 0, acarry = 0;
    int nx[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int64_t i = (int64_t)k * 1024 + tid;
        nx[k] = i < G ? counts[i] : 0;
    }
    for (int64_t base = 0; base < G; base += kScanTile) {
        __syncthreads();
#pragma unroll
        for (int k = 0; k < 4; ++k) tile[k * 1024 + tid] = nx[k];
        const int64_t nb = base + kScanTile;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int64_t i = nb + k * 1024 + tid;
            nx[k] = i < G ? counts[i] : 0;
        }
        __syncthreads();
        int v[4], sum = 0, act = 0;
        for (int k = 0; k < 4; ++k) {
            v[k] = tile[4 * tid + k];
            sum += v[k];
            act += v[k] > 0;
        }
        int total, atotal;
        int run = carry + block_exclusive_scan(sum, sh32, &total);
        int arun = acarry + block_exclusive_scan(act, sh32, &atotal);
        for (int k = 0; k < 4; ++k) {
            const int64_t g = base + 4 * tid + k;
            tile2[4 * tid + k] = run;
            run += v[k];
            if (v[k] > 0 && g < G) active[arun++] = (int32_t)g;
        }
        carry += total;
        acarry += atotal;
        __syncthreads();
        for (int k = 0; k < 4; ++k) {
            const int64_t i = base + k * 1024 + tid;
            if (i < G) {
                offsets[i] = tile2[k * 1024 + tid];
                counts_out[i] = tile[k * 1024 + tid] < 0 ? 0 : counts[i];
            }
        }
    }
    if (tid == 0) {
        offsets[G] = carry;
        *num_active = acarry;
    }
}

// --------------------------------------------------- 3. radix passes
// Exclusive scan of n ints in place, one CTA of 1024 threads; with `tail`,
// the total is written there.
__global__ void __launch_bounds__(1024) exclusive_scan_kernel(int32_t *__restrict__ a,
                                                             int64_t n, int32_t *tail) {
    __shared__ int tile[kScanTile];
    __shared__ int sh32[33];
    grid_dependency_wait();
    grid_dependents_launch();
    cta_exclusive_scan(a, n, tail, tile, sh32);
}

constexpr int kRounds = kItemsPerWarp / 32;                       // 8

// Stable scatter of one tile.  Warp w owns tile items [w*256, (w+1)*256) and
// walks them in rounds of 32, so ranks follow input order.  If hist_next is
// given, the digits of the next pass are counted per output tile.
__global__ void __launch_bounds__(kScatterThreads) radix_scatter_kernel(
    const int32_t *__restrict__ src_tok, const int32_t *__restrict__ src_exp,
    const float *__restrict__ src_gate, int64_t M, int B, int shift, uint32_t dmask,
    int64_t ntiles, const int32_t *__restrict__ hist_scanned, int32_t *__restrict__ dst_tok,
    int32_t *__restrict__ dst_exp, float *__restrict__ dst_gate,
    int32_t *__restrict__ hist_next, int next_shift, uint32_t next_dmask, int agg) {
    __shared__ int wcount[kScatterThreads / 32][256];
    grid_dependency_wait();
    grid_dependents_launch();
    const int tid = threadIdx.x, warp = tid >> 5;
    const unsigned lane = lane_id();
    for (int i = tid; i < (kScatterThreads / 32) * 256; i += kScatterThreads)
        (&wcount[0][0])[i] = 0;
    const int64_t wbase = (int64_t)blockIdx.x * kSortTile + (int64_t)warp * kItemsPerWarp;
    int32_t e[kRounds], tk[kRounds];
    float g[kRounds];
#pragma unroll
    for (int j = 0; j < kRounds; ++j) {
        const int64_t m = wbase + j * 32 + lane;
        const bool valid = m < M;
        e[j] = valid ? src_exp[m] : -1;
        tk[j] = valid ? src_tok[m] : 0;
        g[j] = valid ? src_gate[m] : 0.f;
    }
    __syncthreads();
    // per-warp digit counts
#pragma unroll
    for (int j = 0; j < kRounds; ++j) {
        const bool valid = e[j] >= 0;
        const uint32_t dg = valid ? digit_of(e[j], B, shift, dmask) : 0xffffffffu;
        const unsigned peers = __match_any_sync(0xffffffffu, dg);
        if (valid && (lanemask_lt() & peers) == 0) wcount[warp][dg] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // turn counts into per-warp starting positions
    if ((uint32_t)tid <= dmask) {
        int run = hist_scanned[(int64_t)tid * ntiles + blockIdx.x];
        for (int w = 0; w < kScatterThreads / 32; ++w) {
            const int c = wcount[w][tid];
            wcount[w][tid] = run;
            run += c;
        }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kRounds; ++j) {
        const bool valid = e[j] >= 0;
        const uint32_t dg = valid ? digit_of(e[j], B, shift, dmask) : 0xffffffffu;
        const unsigned peers = __match_any_sync(0xffffffffu, dg);
        int pos = -1;
        if (valid) {
            pos = wcount[warp][dg] + __popc(peers & lanemask_lt());
            dst_tok[pos] = tk[j];
            dst_exp[pos] = e[j];
            dst_gate[pos] = g[j];
        }
        if (hist_next) {
            // the next pass's (digit, output tile) counter; with `agg` (crowded
            // groups put many tasks on one counter) lanes with the same key
            // share one atomic
            const uint32_t hk = valid ? digit_of(e[j], B, next_shift, next_dmask) * (uint32_t)ntiles +
                                            (uint32_t)(pos / kSortTile)
                                      : 0xffffffffu;
            if (agg) {
                const unsigned hp = __match_any_sync(0xffffffffu, hk);
                if (valid && lane == (unsigned)(__ffs(hp) - 1)) atomicAdd(&hist_next[hk], __popc(hp));
            } else if (valid) {
                atomicAdd(&hist_next[hk], 1);
            }
        }
        __syncwarp();
        if (valid && (lanemask_lt() & peers) == 0) wcount[warp][dg] += __popc(peers);
        __syncwarp();
    }
}

}  // namespace

cudaError_t launch_exclusive_scan(int32_t *a, int64_t n, int32_t *total, cudaStream_t st) {
    return launch(exclusive_scan_kernel, dim3(1), dim3(1024), 0, st, a, n, total);
}

namespace {
// Grouping by q = e / B without ordering inside a group (the routed forward's
// schedule, where the expert stage needs each group's tasks together but in
// no particular order): task i of the token-order arrays goes to
// offsets[q] + (a position counted down from the group's total in counts[q]).
// Lanes of a warp with the same q (a warp holds a quarter to all of one
// token's tasks) share one atomic and keep their order.  A position outside the
// group's range (counts that do not match the tasks) is reported as
// OMNI_DEV_BAD_SCHEDULE and not written.
__global__ void __launch_bounds__(kScatterThreads) group_scatter_kernel(
    const int32_t *__restrict__ a_tok, const int32_t *__restrict__ a_exp,
    const float *__restrict__ a_gate, int64_t M, int B, int64_t G,
    const int32_t *__restrict__ offsets, int32_t *__restrict__ counts, int32_t *__restrict__ d_tok,
    int32_t *__restrict__ d_exp, float *__restrict__ d_gate, int *status) {
    grid_dependency_wait();
    grid_dependents_launch();
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const unsigned lane = lane_id();
    int32_t t = 0, e = 0;
    float g = 0.f;
    int64_t q = -1;
    if (i < M) {
        t = a_tok[i];
        e = a_exp[i];
        g = a_gate[i];
        q = e >= 0 ? e / B : -1;
        if (q >= G) q = -1;
        if (q < 0) set_status(status, OMNI_DEV_BAD_EXPERT);
    }
    const unsigned peers = __match_any_sync(0xffffffffu, (unsigned)(q + 1));
    const int leader = __ffs(peers) - 1;
    const int n = __popc(peers);
    int base = 0;
    if (q >= 0 && (int)lane == leader) base = atomicSub(&counts[q], n) - n;
    base = __shfl_sync(0xffffffffu, base, leader);
    if (q >= 0) {
        const int r = base + __popc(peers & lanemask_lt());
        const int64_t o0 = offsets[q], o1 = offsets[q + 1];
        const int64_t pos = o0 + r;
        if (r < 0 || pos >= o1) {
            set_status(status, OMNI_DEV_BAD_SCHEDULE);
        } else {
            d_tok[pos] = t;
            d_exp[pos] = e;
            d_gate[pos] = g;
        }
    }
}

// The same scatter for crowded groups (a few groups hold thousands of tasks):
// a CTA of 1024 threads first gathers its tasks' groups in a shared-memory
// hash table (kAggSlots open-addressed slots, at most 1024 keys), each task
// taking its rank inside the CTA's share of its group; then one thread per
// distinct group takes the CTA's share from counts[q] with one atomic, so a
// hot group's counter sees one atomic per CTA instead of one per warp.
constexpr int kAggThreads = 1024;
constexpr int kAggSlots = 2048;
__global__ void __launch_bounds__(kAggThreads) group_scatter_agg_kernel(
    const int32_t *__restrict__ a_tok, const int32_t *__restrict__ a_exp,
    const float *__restrict__ a_gate, int64_t M, int B, int64_t G,
    const int32_t *__restrict__ offsets, int32_t *__restrict__ counts, int32_t *__restrict__ d_tok,
    int32_t *__restrict__ d_exp, float *__restrict__ d_gate, int *status) {
    __shared__ int keys[kAggSlots];
    __shared__ int cnt[kAggSlots];
    __shared__ int base[kAggSlots];
    grid_dependency_wait();
    grid_dependents_launch();
    for (int h = threadIdx.x; h < kAggSlots; h += kAggThreads) {
        keys[h] = -1;
        cnt[h] = 0;
    }
    const int64_t i = (int64_t)blockIdx.x * kAggThreads + threadIdx.x;
    int32_t t = 0, e = 0;
    float g = 0.f;
    int q = -1;
    if (i < M) {
        t = a_tok[i];
        e = a_exp[i];
        g = a_gate[i];
        const int64_t qq = e >= 0 ? e / B : -1;
        q = qq < G ? (int)qq : -1;
        if (q < 0) set_status(status, OMNI_DEV_BAD_EXPERT);
    }
    __syncthreads();
    int slot = -1, r = 0;
    if (q >= 0) {
        // at most kAggThreads keys in kAggSlots slots: the probe ends
        int h = (int)(((uint32_t)q * 2654435761u) >> 21);          // 11 bits
        for (int probe = 0; probe < kAggSlots; ++probe) {
            const int k = atomicCAS(&keys[h], -1, q);
            if (k == -1 || k == q) {
                slot = h;
                break;
            }
            h = (h + 1) & (kAggSlots - 1);
        }
        if (slot >= 0) r = atomicAdd(&cnt[slot], 1);
    }
    __syncthreads();
    for (int h = threadIdx.x; h < kAggSlots; h += kAggThreads) {
        const int c = cnt[h];
        if (c > 0) base[h] = atomicSub(&counts[keys[h]], c) - c;
    }
    __syncthreads();
    if (slot >= 0) {
        const int64_t o0 = offsets[q], o1 = offsets[q + 1];
        const int rr = base[slot] + r;
        const int64_t pos = o0 + rr;
        if (rr < 0 || pos >= o1) {
            set_status(status, OMNI_DEV_BAD_SCHEDULE);
        } else {
            d_tok[pos] = t;
            d_exp[pos] = e;
            d_gate[pos] = g;
        }
    }
}
}  // namespace

int sched_pass_width(const Sizes &sz) {
    return sz.passes ? (sz.qbits + sz.passes - 1) / sz.passes : 0;
}

uint32_t sched_pass_mask(const Sizes &sz, int p) {
    const int width = sched_pass_width(sz);
    const int shift = p * width;
    const int w = (sz.qbits - shift) < width ? (sz.qbits - shift) : width;
    return (1u << w) - 1u;
}

bool sched_aggregate(const Sizes &sz) {
    // crowded groups (64 tasks or more per group on average): the radix
    // histogram atomics would pile up on a few addresses, so warps combine
    // equal ones first
    return sz.M >= 64 * sz.G;
}

// Grouping only whenever there is more than one group.  Measured on B200 it
// also wins where groups are crowded (a warp's run of equal groups shares one
// cursor atomic): skewed layer 1.152 -> 1.055 ms, L = 65536 8.82 -> 8.56 ms.
bool sched_unordered(const Sizes &sz) { return sz.passes > 0; }

SchedPrep sched_prep_of(const Sizes &sz, void *ws, const WsLayout &lay) {
    SchedPrep o;
    o.a_tok = ws_at<int32_t>(ws, lay.a_tok);
    o.a_exp = ws_at<int32_t>(ws, lay.a_exp);
    o.a_gate = ws_at<float>(ws, lay.a_gate);
    o.counts = ws_at<int32_t>(ws, lay.z_cnt);
    o.bitmap = ws_at<uint32_t>(ws, lay.bitmap);
    o.num_distinct = ws_at<int32_t>(ws, lay.z_ndist);
    o.hist0 = sz.passes ? ws_at<int32_t>(ws, lay.hist) : nullptr;
    o.ntiles = sz.ntiles;
    o.dmask0 = sz.passes ? sched_pass_mask(sz, 0) : 0u;
    o.B = sz.B;
    o.unordered = 0;
    return o;
}

cudaError_t launch_schedule(const int32_t *idx, const float *gate, const Sizes &sz,
                            int32_t *task_token, int32_t *task_expert, float *task_gate,
                            int32_t *group_offsets, int32_t *group_counts,
                            int32_t *active_groups, int32_t *num_active, int32_t *num_distinct,
                            void *ws, const WsLayout &lay, cudaStream_t st, bool prepared,
                            bool any_order) {
    // The caller has zeroed [0, lay.zero_end) of ws: the status word, the
    // group counters, the distinct-expert counter, the bitmap and the radix
    // histograms.  With `prepared`, the per-token step (sched_token.cuh) has
    // already run inside the router's merge kernel.
    const int64_t M = sz.M, G = sz.G;
    int *status = ws_at<int>(ws, lay.hdr);
    int32_t *a_tok = ws_at<int32_t>(ws, lay.a_tok), *a_exp = ws_at<int32_t>(ws, lay.a_exp);
    float *a_gate = ws_at<float>(ws, lay.a_gate);
    int32_t *b_tok = ws_at<int32_t>(ws, lay.b_tok), *b_exp = ws_at<int32_t>(ws, lay.b_exp);
    float *b_gate = ws_at<float>(ws, lay.b_gate);
    int32_t *counts = ws_at<int32_t>(ws, lay.z_cnt);
    int32_t *ndist = ws_at<int32_t>(ws, lay.z_ndist);
    uint32_t *bitmap = ws_at<uint32_t>(ws, lay.bitmap);
    int32_t *hist = ws_at<int32_t>(ws, lay.hist);
    const int64_t ntiles = sz.ntiles;
    const int64_t hstride = 256 * ntiles;                // one histogram per pass
    cudaError_t e;

    // radix passes over q = e / B, digits of at most 8 bits
    const int passes = sz.passes;
    const int width = sched_pass_width(sz);
    auto pass_mask = [&](int p) -> uint32_t { return sched_pass_mask(sz, p); };

    if (!prepared) {
        const int wpb = 8;
        const size_t smem = sizeof(int32_t) * (size_t)sz.K * wpb;
        e = launch(sched_prepare_kernel, dim3((unsigned)((sz.L + wpb - 1) / wpb)), dim3(32 * wpb),
                   smem, st, idx, gate, sz.L, sz.K, (int)sz.N, sz.B, a_tok, a_exp, a_gate, counts,
                   bitmap, ndist, passes ? hist : nullptr, ntiles, passes ? pass_mask(0) : 0u,
                   status);
        if (e != cudaSuccess) return e;
    }
    if (any_order && sched_unordered(sz)) {
        // grouping only: offsets, then one scatter that counts each group's
        // tasks down from its total (the counters are not needed after the scan)
        e = launch(sched_scan_kernel, dim3(1), dim3(1024), 0, st, counts, G, group_counts,
                   group_offsets, active_groups, num_active, ndist, num_distinct,
                   (int32_t *)nullptr, (int64_t)0);
        if (e != cudaSuccess) return e;
        if (sched_aggregate(sz)) {
            const unsigned grid = (unsigned)((M + kAggThreads - 1) / kAggThreads);
            return launch(group_scatter_agg_kernel, dim3(grid), dim3(kAggThreads), 0, st, a_tok,
                          a_exp, a_gate, M, sz.B, G, (const int32_t *)group_offsets, counts,
                          task_token, task_expert, task_gate, status);
        }
        const unsigned grid = (unsigned)((M + kScatterThreads - 1) / kScatterThreads);
        return launch(group_scatter_kernel, dim3(grid), dim3(kScatterThreads), 0, st, a_tok, a_exp,
                      a_gate, M, sz.B, G, (const int32_t *)group_offsets, counts, task_token,
                      task_expert, task_gate, status);
    }
    e = launch(sched_scan_kernel, dim3(passes ? 2 : 1), dim3(1024), 0, st, counts, G,
               group_counts, group_offsets, active_groups, num_active, ndist, num_distinct, hist,
               passes ? (int64_t)(pass_mask(0) + 1) * ntiles : (int64_t)0);
    if (e != cudaSuccess) return e;

    if (passes == 0) {
        if ((e = cudaMemcpyAsync(task_token, a_tok, 4 * M, cudaMemcpyDeviceToDevice, st))) return e;
        if ((e = cudaMemcpyAsync(task_expert, a_exp, 4 * M, cudaMemcpyDeviceToDevice, st))) return e;
        e = cudaMemcpyAsync(task_gate, a_gate, 4 * M, cudaMemcpyDeviceToDevice, st);
        first_launch_in_call();         // a kernel after these copies must not overlap them
        return e;
    }
    const int32_t *s_tok = a_tok, *s_exp = a_exp;
    const float *s_gate = a_gate;
    for (int p = 0; p < passes; ++p) {
        const int shift = p * width;
        const uint32_t dmask = pass_mask(p);
        const bool last = p == passes - 1;
        int32_t *h = hist + hstride * p;
        if (p > 0) {
            e = launch(exclusive_scan_kernel, dim3(1), dim3(1024), 0, st, h,
                       (int64_t)(dmask + 1) * ntiles, (int32_t *)nullptr);
            if (e != cudaSuccess) return e;
        }
        // ping-pong: the last pass writes the caller's arrays
        int32_t *d_tok, *d_exp;
        float *d_gate;
        if (last) {
            d_tok = task_token; d_exp = task_expert; d_gate = task_gate;
        } else if (s_tok == a_tok) {
            d_tok = b_tok; d_exp = b_exp; d_gate = b_gate;
        } else {
            d_tok = a_tok; d_exp = a_exp; d_gate = a_gate;
        }
        e = launch(radix_scatter_kernel, dim3((unsigned)ntiles), dim3(kScatterThreads), 0, st,
                   s_tok, s_exp, s_gate, M, sz.B, shift, dmask, ntiles, (const int32_t *)h, d_tok,
                   d_exp, d_gate, last ? nullptr : hist + hstride * (p + 1), (p + 1) * width,
                   last ? 0u : pass_mask(p + 1), sched_aggregate(sz) ? 1 : 0);
        if (e != cudaSuccess) return e;
        s_tok = d_tok; s_exp = d_exp; s_gate = d_gate;
    }
    return cudaSuccess;
}

}  // namespace omni

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
//      them in (t, e) order, count tasks per group, mark experts in a bitmap.
//   2. group scan (1 CTA): exclusive scan of the group counts, active-group
//      list, number of distinct experts.
//   3. LSD radix sort of the tasks on q alone, 8-bit digits, stable.  The
//      input is in (t, e) order, so a stable sort by q yields (q, t, e).
//      Each pass: per-tile digit histogram, one exclusive scan, stable scatter
//      (warps rank equal digits with __match_any_sync, in input order).
#include "omni_common.cuh"
#include "omni_internal.h"

namespace omni {
namespace {

constexpr int kScatterThreads = 256;                       // 8 warps
constexpr int kItemsPerWarp = kSortTile / (kScatterThreads / 32);   // 256

// ---------------------------------------------------------- 1. prepare
__global__ void sched_prepare_kernel(const int32_t *__restrict__ idx,
                                     const float *__restrict__ gate, int L, int K, int N, int B,
                                     int32_t *__restrict__ a_tok, int32_t *__restrict__ a_exp,
                                     float *__restrict__ a_gate, int32_t *__restrict__ counts,
                                     uint32_t *__restrict__ bitmap, int *status) {
    extern __shared__ int32_t sh_e[];
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
    for (int u = lane; u < K; u += 32) {
        const int32_t eu = e_s[u];
        int r = 0;
        for (int v = 0; v < K; ++v) {
            const int32_t ev = e_s[v];
            r += (ev < eu) | ((ev == eu) & (v < u));
        }
        const float g = (idx[row + u] < 0 || idx[row + u] >= N) ? 0.f : gate[row + u];
        a_tok[row + r] = t;
        a_exp[row + r] = eu;
        a_gate[row + r] = g;
        atomicAdd(&counts[eu / B], 1);
        atomicOr(&bitmap[eu >> 5], 1u << (eu & 31));
    }
}

// ----------------------------------------------------- 2. group scan
// One CTA of 1024 threads; thread t owns a contiguous chunk of groups.
__global__ void __launch_bounds__(1024) sched_group_scan_kernel(
    const int32_t *__restrict__ counts, int64_t G, const uint32_t *__restrict__ bitmap,
    int64_t nwords, int32_t *__restrict__ offsets, int32_t *__restrict__ active,
    int32_t *__restrict__ num_active, int32_t *__restrict__ num_distinct) {
    __shared__ int sh_sum[32], sh_act[32], sh_pop[32];
    const int tid = threadIdx.x;
    const int64_t per = (G + 1023) / 1024;
    const int64_t g0 = (int64_t)tid * per;
    const int64_t g1 = g0 + per < G ? g0 + per : G;
    int sum = 0, act = 0, pop = 0;
    for (int64_t g = g0; g < g1; ++g) {
        const int c = counts[g];
        sum += c;
        act += c > 0;
    }
    for (int64_t w = tid; w < nwords; w += 1024) pop += __popc(bitmap[w]);
    // block exclusive scans of sum and act, block sum of pop
    const int lane = tid & 31, warp = tid >> 5;
    const int isum = warp_iscan(sum), iact = warp_iscan(act);
    const int wpop = warp_isum(pop);
    if (lane == 31) {
        sh_sum[warp] = isum;
        sh_act[warp] = iact;
    }
    if (lane == 0) sh_pop[warp] = wpop;
    __syncthreads();
    if (warp == 0) {
        const int s = sh_sum[lane], a = sh_act[lane], p = sh_pop[lane];
        const int is = warp_iscan(s), ia = warp_iscan(a), ps = warp_isum(p);
        sh_sum[lane] = is - s;
        sh_act[lane] = ia - a;
        if (lane == 31) {
            offsets[G] = is;
            *num_active = ia;
        }
        if (lane == 0) *num_distinct = ps;
    }
    __syncthreads();
    int run = sh_sum[warp] + isum - sum;
    int arun = sh_act[warp] + iact - act;
    for (int64_t g = g0; g < g1; ++g) {
        const int c = counts[g];
        offsets[g] = run;
        run += c;
        if (c > 0) active[arun++] = (int32_t)g;
    }
}

// --------------------------------------------------- 3. radix passes
__device__ __forceinline__ uint32_t digit_of(int32_t e, int B, int shift, uint32_t dmask) {
    return ((uint32_t)(e / B) >> shift) & dmask;
}

__global__ void __launch_bounds__(kScatterThreads) radix_hist_kernel(
    const int32_t *__restrict__ src_exp, int64_t M, int B, int shift, uint32_t dmask,
    int64_t ntiles, int32_t *__restrict__ hist) {
    __shared__ int h[256];
    const int tid = threadIdx.x;
    h[tid] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kSortTile;
    for (int i = tid; i < kSortTile; i += kScatterThreads) {
        const int64_t m = base + i;
        if (m < M) atomicAdd(&h[digit_of(src_exp[m], B, shift, dmask)], 1);
    }
    __syncthreads();
    if ((uint32_t)tid <= dmask) hist[(int64_t)tid * ntiles + blockIdx.x] = h[tid];
}

// Exclusive scan of n ints in place, one CTA of 1024 threads.
__global__ void __launch_bounds__(1024) exclusive_scan_kernel(int32_t *__restrict__ a,
                                                             int64_t n) {
    __shared__ int sh[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t per = (n + 1023) / 1024;
    const int64_t i0 = (int64_t)tid * per;
    const int64_t i1 = i0 + per < n ? i0 + per : n;
    int sum = 0;
    for (int64_t i = i0; i < i1; ++i) sum += a[i];
    const int incl = warp_iscan(sum);
    if (lane == 31) sh[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int s = sh[lane];
        sh[lane] = warp_iscan(s) - s;
    }
    __syncthreads();
    int run = sh[warp] + incl - sum;
    for (int64_t i = i0; i < i1; ++i) {
        const int v = a[i];
        a[i] = run;
        run += v;
    }
}

// Stable scatter of one tile.  Warp w owns tile items [w*256, (w+1)*256) and
// walks them in rounds of 32, so ranks follow input order.
__global__ void __launch_bounds__(kScatterThreads) radix_scatter_kernel(
    const int32_t *__restrict__ src_tok, const int32_t *__restrict__ src_exp,
    const float *__restrict__ src_gate, int64_t M, int B, int shift, uint32_t dmask,
    int64_t ntiles, const int32_t *__restrict__ hist_scanned, int32_t *__restrict__ dst_tok,
    int32_t *__restrict__ dst_exp, float *__restrict__ dst_gate) {
    __shared__ int wcount[kScatterThreads / 32][256];
    const int tid = threadIdx.x, warp = tid >> 5;
    const unsigned lane = lane_id();
    for (int i = tid; i < (kScatterThreads / 32) * 256; i += kScatterThreads)
        (&wcount[0][0])[i] = 0;
    __syncthreads();
    const int64_t wbase = (int64_t)blockIdx.x * kSortTile + (int64_t)warp * kItemsPerWarp;
    // per-warp digit counts
    for (int j = 0; j < kItemsPerWarp; j += 32) {
        const int64_t m = wbase + j + lane;
        const bool valid = m < M;
        const uint32_t dg = valid ? digit_of(src_exp[m], B, shift, dmask) : 0xffffffffu;
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
    for (int j = 0; j < kItemsPerWarp; j += 32) {
        const int64_t m = wbase + j + lane;
        const bool valid = m < M;
        int32_t e = 0, tk = 0;
        float g = 0.f;
        if (valid) {
            e = src_exp[m];
            tk = src_tok[m];
            g = src_gate[m];
        }
        const uint32_t dg = valid ? digit_of(e, B, shift, dmask) : 0xffffffffu;
        const unsigned peers = __match_any_sync(0xffffffffu, dg);
        if (valid) {
            const int pos = wcount[warp][dg] + __popc(peers & lanemask_lt());
            dst_tok[pos] = tk;
            dst_exp[pos] = e;
            dst_gate[pos] = g;
        }
        __syncwarp();
        if (valid && (lanemask_lt() & peers) == 0) wcount[warp][dg] += __popc(peers);
        __syncwarp();
    }
}

}  // namespace

cudaError_t launch_schedule(const int32_t *idx, const float *gate, const Sizes &sz,
                            int32_t *task_token, int32_t *task_expert, float *task_gate,
                            int32_t *group_offsets, int32_t *group_counts,
                            int32_t *active_groups, int32_t *num_active, int32_t *num_distinct,
                            void *ws, const WsLayout &lay, cudaStream_t st) {
    const int64_t M = sz.M, G = sz.G;
    int *status = ws_at<int>(ws, lay.hdr);
    int32_t *a_tok = ws_at<int32_t>(ws, lay.a_tok), *a_exp = ws_at<int32_t>(ws, lay.a_exp);
    float *a_gate = ws_at<float>(ws, lay.a_gate);
    int32_t *b_tok = ws_at<int32_t>(ws, lay.b_tok), *b_exp = ws_at<int32_t>(ws, lay.b_exp);
    float *b_gate = ws_at<float>(ws, lay.b_gate);
    uint32_t *bitmap = ws_at<uint32_t>(ws, lay.bitmap);
    int32_t *hist = ws_at<int32_t>(ws, lay.hist);
    const int64_t nwords = (sz.N + 31) / 32;
    cudaError_t e;

    if ((e = cudaMemsetAsync(group_counts, 0, sizeof(int32_t) * G, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(bitmap, 0, sizeof(uint32_t) * nwords, st)) != cudaSuccess) return e;
    {
        const int wpb = 8;
        const size_t smem = sizeof(int32_t) * (size_t)sz.K * wpb;
        sched_prepare_kernel<<<(unsigned)((sz.L + wpb - 1) / wpb), 32 * wpb, smem, st>>>(
            idx, gate, sz.L, sz.K, (int)sz.N, sz.B, a_tok, a_exp, a_gate, group_counts, bitmap,
            status);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    sched_group_scan_kernel<<<1, 1024, 0, st>>>(group_counts, G, bitmap, nwords, group_offsets,
                                                 active_groups, num_active, num_distinct);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    // radix passes over q = e / B
    int nbits = 0;
    while (nbits < 31 && ((int64_t)1 << nbits) < G) ++nbits;       // bits of G - 1
    const int passes = (nbits + 7) / 8;
    if (passes == 0) {
        if ((e = cudaMemcpyAsync(task_token, a_tok, 4 * M, cudaMemcpyDeviceToDevice, st))) return e;
        if ((e = cudaMemcpyAsync(task_expert, a_exp, 4 * M, cudaMemcpyDeviceToDevice, st))) return e;
        return cudaMemcpyAsync(task_gate, a_gate, 4 * M, cudaMemcpyDeviceToDevice, st);
    }
    const int width = (nbits + passes - 1) / passes;
    const int64_t ntiles = sz.ntiles;
    const int32_t *s_tok = a_tok, *s_exp = a_exp;
    const float *s_gate = a_gate;
    for (int p = 0; p < passes; ++p) {
        const int shift = p * width;
        const int w = (nbits - shift) < width ? (nbits - shift) : width;
        const uint32_t dmask = (1u << w) - 1u;
        const bool last = p == passes - 1;
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
        radix_hist_kernel<<<(unsigned)ntiles, kScatterThreads, 0, st>>>(s_exp, M, sz.B, shift,
                                                                         dmask, ntiles, hist);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        exclusive_scan_kernel<<<1, 1024, 0, st>>>(hist, (int64_t)(dmask + 1) * ntiles);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        radix_scatter_kernel<<<(unsigned)ntiles, kScatterThreads, 0, st>>>(
            s_tok, s_exp, s_gate, M, sz.B, shift, dmask, ntiles, hist, d_tok, d_exp, d_gate);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        s_tok = d_tok; s_exp = d_exp; s_gate = d_gate;
    }
    return cudaSuccess;
}

}  // namespace omni

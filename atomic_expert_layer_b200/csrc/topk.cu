// topk.cu -- Cartesian product router selection on sm_100a.
//
// "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale"
// (rainbus review page, method paragraph, step 2): p_r, p_c are the
// LogSoftmax of the row and column logits and the score of expert (i, j) is
// S_ij = p_r[i] + p_c[j]; the global top-K is taken without building the
// N_r x N_c grid.  The order key is (S desc, p_r desc, p_c desc, n asc) with
// n = i * N_c + j, and axis ranks use (p desc, index asc).  Gates are the
// softmax over the K selected scores.
//
// Kernel 1 (axis_topk): one warp per (token, axis).  Optional LogSoftmax
//   (from the router GEMM's per-tile max / sum-exp partials when given),
//   then the axis' top min(K, n) entries.
// Kernel 2 (merge_topk): one warp per token.  Because fp32 addition is
//   monotone, a cell with row rank a and column rank b is dominated by every
//   cell (a', b') with a' <= a, b' <= b, and the key above ranks a dominating
//   cell first even on equal S; so the K best cells all satisfy
//   (a+1)(b+1) <= K.  Those C candidates (C = sum_a min(Kc, K/(a+1))) are
//   scored and the K best taken.
//
// Selection (both kernels, exact): values are bucketed by
//   b(v) = floor((vmax - v) * 32)       (fp32, monotone non-increasing in v)
// over 256 buckets (8 units below the maximum).  Any value in a lower
// bucket is strictly larger than any value in a higher one, so with b* the
// bucket holding the k-th value, the top k are all values with b < b* plus
// the best of bucket b*.  Those candidates (about k + 1 for Gaussian-like
// rows) are placed by a counting sort on the bucket (buckets are in value
// order) and ranked by the full key only among the peers of their bucket.
// If fewer than k values lie within 8 units of the maximum, or there are
// more candidates than the kernel's capacity, an exact radix select (4
// passes of 8 bits over order-preserving keys) followed by a rank sort is
// used instead.
#include <cstring>

#include "omni_common.cuh"
#include "omni_internal.h"
#include "router_small.cuh"
#include "sched_token.cuh"

namespace omni {
namespace {

constexpr int kNB = 256;               // value buckets (also the radix histogram)
constexpr float kBucketScale = 32.f;   // buckets per unit: 8 units below the maximum

// ----------------------------------------------------------- radix select
// Exact k-th largest key of keys[0..n) (a warp, smem histogram `hist` of 256).
// Returns the threshold key T and sets *take_eq to how many keys equal to T
// belong to the top k (the rest of the top k is every key > T).
__device__ uint32_t warp_radix_select(const uint32_t *keys, int n, int k, uint32_t *hist,
                                      int *take_eq) {
    const unsigned lane = lane_id();
    uint32_t prefix = 0, mask = 0;
    int krem = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = lane; b < 256; b += 32) hist[b] = 0;
        __syncwarp();
        for (int i = lane; i < n; i += 32) {
            const uint32_t key = keys[i];
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncwarp();
        // lane l owns bins 255-8l down to 248-8l
        int c[8], tot = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            c[j] = (int)hist[255 - 8 * lane - j];
            tot += c[j];
        }
        const int incl = warp_iscan(tot);
        const int excl = incl - tot;
        const bool mine = excl < krem && krem <= incl;
        const unsigned bal = __ballot_sync(0xffffffffu, mine);
        int digit = 0, above = 0;
        if (mine) {
            int run = excl;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (run + c[j] >= krem) {
                    digit = 255 - 8 * (int)lane - j;
                    above = run;
                    break;
                }
                run += c[j];
            }
        }
        const int src = __ffs(bal) - 1;
        digit = __shfl_sync(0xffffffffu, digit, src);
        above = __shfl_sync(0xffffffffu, above, src);
        krem -= above;
        prefix |= (uint32_t)digit << shift;
        mask |= 255u << shift;
        __syncwarp();
    }
    *take_eq = krem;
    return prefix;
}

// ------------------------------------------------------------ value buckets
__device__ __forceinline__ int bucket_of(float vmax, float v) {
    const float dv = __fmul_rn(__fsub_rn(vmax, v), kBucketScale);
    return dv < (float)kNB ? (int)dv : kNB;           // kNB = beyond the range
}

// Find the bucket b* holding the k-th largest value from a filled histogram.
// Returns the number of values in buckets <= b*, or -1 if fewer than k values
// are in range.
__device__ int bucket_find(const uint32_t *hist, int k, int *bstar) {
    const unsigned lane = lane_id();
    constexpr int per = kNB / 32;            // lane l owns buckets [l * per, (l + 1) * per)
    int tot = 0;
#pragma unroll
    for (int j = 0; j < per; ++j) tot += (int)hist[lane * per + j];
    const int incl = warp_iscan(tot);
    const int excl = incl - tot;
    const bool mine = excl < k && k <= incl;
    const unsigned bal = __ballot_sync(0xffffffffu, mine);
    if (bal == 0u) return -1;
    int bs = 0, through = 0;
    if (mine) {
        int run = excl;
#pragma unroll
        for (int j = 0; j < per; ++j) {
            run += (int)hist[lane * per + j];
            if (run >= k && through == 0) {
                bs = lane * per + j;
                through = run;
            }
        }
    }
    const int src = __ffs(bal) - 1;
    *bstar = __shfl_sync(0xffffffffu, bs, src);
    return __shfl_sync(0xffffffffu, through, src);
}

// Zero the histogram, count get(0..n) into it and find b* (see bucket_find).
template <typename Get>
__device__ int bucket_threshold(Get get, int n, int k, float vmax, uint32_t *hist, int *bstar) {
    const unsigned lane = lane_id();
    for (int b = lane; b < kNB; b += 32) hist[b] = 0u;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
        const int b = bucket_of(vmax, get(i));
        if (b < kNB) atomicAdd(&hist[b], 1u);
    }
    __syncwarp();
    return bucket_find(hist, k, bstar);
}

// LogSoftmax normaliser of row t from the router GEMM's partials: per 64
// columns (max, sum exp(s - max)).  Returns lse; *mx is the row maximum.
__device__ __forceinline__ float lse_from_partials(const float2 *part, int t, int n, float *mx_out) {
    const unsigned lane = lane_id();
    const int nt = 2 * ((n + 2 * kGemmPartCols - 1) / (2 * kGemmPartCols));
    float m = -INFINITY, sm_ = 0.f;
    for (int u = lane; u < nt; u += 32) {
        const float2 pt = part[(size_t)t * nt + u];
        if (pt.x > -INFINITY) {
            const float mn = fmaxf(m, pt.x);
            sm_ = (m > -INFINITY ? sm_ * __expf(m - mn) : 0.f) + pt.y * __expf(pt.x - mn);
            m = mn;
        }
    }
    const float mx = warp_max(m);
    float sum = (m > -INFINITY) ? sm_ * __expf(m - mx) : 0.f;
    sum = warp_sum(sum);
    *mx_out = mx;
    return mx + __logf(sum);
}

// --------------------------------------------------- bucket counting sort
// After bucket_threshold: turn the counts of buckets [0, kNB) into starting
// positions (exclusive prefix, written back into hist) and copy them to cur.
__device__ __forceinline__ void bucket_starts(uint32_t *hist, uint32_t *cur) {
    const unsigned lane = lane_id();
    constexpr int per = kNB / 32;
    uint32_t c[per];
    int tot = 0;
#pragma unroll
    for (int j = 0; j < per; ++j) {
        c[j] = hist[lane * per + j];
        tot += (int)c[j];
    }
    int run = warp_iscan(tot) - tot;
#pragma unroll
    for (int j = 0; j < per; ++j) {
        hist[lane * per + j] = (uint32_t)run;
        cur[lane * per + j] = (uint32_t)run;
        run += (int)c[j];
    }
    __syncwarp();
}

// bucket_find and bucket_starts in one pass over the histogram (one warp):
// the counts become starting positions (written to hist and cur), and the
// return value / *bstar are those of bucket_find.
__device__ int bucket_scan(uint32_t *hist, uint32_t *cur, int k, int *bstar) {
    const unsigned lane = lane_id();
    constexpr int per = kNB / 32;
    uint32_t c[per];
    int tot = 0;
#pragma unroll
    for (int j = 0; j < per; ++j) {
        c[j] = hist[lane * per + j];
        tot += (int)c[j];
    }
    const int incl = warp_iscan(tot);
    const int excl = incl - tot;
    const bool mine = excl < k && k <= incl;
    const unsigned bal = __ballot_sync(0xffffffffu, mine);
    int run = excl, bs = 0, through = 0;
#pragma unroll
    for (int j = 0; j < per; ++j) {
        hist[lane * per + j] = (uint32_t)run;
        cur[lane * per + j] = (uint32_t)run;
        run += (int)c[j];
        if (mine && through == 0 && run >= k) {
            bs = lane * per + j;
            through = run;
        }
    }
    if (bal == 0u) return -1;
    const int src = __ffs(bal) - 1;
    *bstar = __shfl_sync(0xffffffffu, bs, src);
    return __shfl_sync(0xffffffffu, through, src);
}

// ------------------------------------------------------------ axis top-K
// Dynamic smem per warp (words): vals[nmax] | hist[kNB] | cur[kNB] |
// area[max(2 kmax, 2 CAP)], where area is either sel_key[kmax] + sel_idx[kmax]
// (fallback) or the candidate keys tmp[CAP] (u64)
// One (token, axis) row, one warp, exact: LogSoftmax (optional; from the
// GEMM partials when given) and the top kx = min(K, n) of the row by
// (p desc, index asc) into oval / oidx.  `base` is the warp's shared area of
// nmax + 2 kNB + 2 kmax (+1) words.
template <int CAP>
__device__ void axis_row_exact(const float *__restrict__ in, int n, int kx, int logsoftmax,
                               const float2 *__restrict__ part, int t, float *__restrict__ pout,
                               float *__restrict__ oval, int *__restrict__ oidx, int nmax,
                               int kmax, uint32_t *base) {
    const unsigned lane = lane_id();
    float *vals = reinterpret_cast<float *>(base);
    uint32_t *hist = base + nmax;
    uint32_t *cur = hist + kNB;
    const size_t area_off = ((size_t)nmax + 2 * kNB + 1) & ~(size_t)1;  // 8-byte aligned
    uint32_t *sel_key = base + area_off;
    int *sel_idx = reinterpret_cast<int *>(sel_key + kmax);
    uint64_t *tmp = reinterpret_cast<uint64_t *>(base + area_off);

    float vmax = -INFINITY;
    bool counted = false;                  // buckets already filled
    if (logsoftmax && part) {
        float mx;
        const float lse = lse_from_partials(part, t, n, &mx);
        vmax = mx - lse;                   // the p of the largest logit, same rounding
        if (CAP > 0) {
            for (int b = lane; b < kNB; b += 32) hist[b] = 0u;
            __syncwarp();
        }
        // one pass: p = s - lse, kept in shared memory, counted into the buckets
        auto count = [&](float p) {
            if (CAP > 0) {
                const int b = bucket_of(vmax, p);
                if (b < kNB) atomicAdd(&hist[b], 1u);
            }
        };
        if ((n & 3) == 0 && (reinterpret_cast<uintptr_t>(in) & 15u) == 0) {
            // 16-byte loads and 16-byte shared stores (no bank conflicts)
            const float4 *in4 = reinterpret_cast<const float4 *>(in);
            float4 *v4 = reinterpret_cast<float4 *>(vals);
            float *prow = pout ? pout + (size_t)t * n : nullptr;
            const bool o_vec = prow && (reinterpret_cast<uintptr_t>(prow) & 15u) == 0;
            float4 *o4 = reinterpret_cast<float4 *>(prow);
            const int n4 = n >> 2;
#pragma unroll 4
            for (int i4 = lane; i4 < n4; i4 += 32) {
                const float4 v = in4[i4];
                const float4 p = make_float4(v.x - lse, v.y - lse, v.z - lse, v.w - lse);
                v4[i4] = p;
                if (o_vec) {
                    o4[i4] = p;
                } else if (prow) {
                    prow[4 * i4] = p.x;
                    prow[4 * i4 + 1] = p.y;
                    prow[4 * i4 + 2] = p.z;
                    prow[4 * i4 + 3] = p.w;
                }
                count(p.x);
                count(p.y);
                count(p.z);
                count(p.w);
            }
        } else {
#pragma unroll 4
            for (int i = lane; i < n; i += 32) {
                const float p = in[i] - lse;
                if (pout) pout[(size_t)t * n + i] = p;
                vals[i] = p;
                count(p);
            }
        }
        counted = true;
    } else if (logsoftmax) {
        // the row into shared memory with every load in flight (16-byte
        // vectors when the row allows), then the max over the stored values
        if ((n & 3) == 0 && (reinterpret_cast<uintptr_t>(in) & 15u) == 0) {
            const float4 *in4 = reinterpret_cast<const float4 *>(in);
            float4 *v4 = reinterpret_cast<float4 *>(vals);
            const int n4 = n >> 2;
#pragma unroll 8
            for (int i4 = lane; i4 < n4; i4 += 32) v4[i4] = in4[i4];
        } else {
#pragma unroll 8
            for (int i = lane; i < n; i += 32) vals[i] = in[i];
        }
        __syncwarp();
        float mx = -INFINITY;
        for (int i = lane; i < n; i += 32) mx = fmaxf(mx, vals[i]);
        mx = warp_max(mx);
        float sum = 0.f;
        for (int i = lane; i < n; i += 32) sum += __expf(vals[i] - mx);
        sum = warp_sum(sum);
        const float lse = mx + __logf(sum);
        for (int i = lane; i < n; i += 32) {
            const float p = vals[i] - lse;
            if (pout) pout[(size_t)t * n + i] = p;
            vals[i] = p;
        }
        vmax = mx - lse;                   // the p of the largest logit, same rounding
    } else {
        for (int i = lane; i < n; i += 32) {
            const float v = in[i];
            vals[i] = v;
            vmax = fmaxf(vmax, v);
        }
        vmax = warp_max(vmax);
    }
    __syncwarp();

    if (CAP > 0) {
        int bs = 0;
        const int ncand =
            counted ? bucket_find(hist, kx, &bs)
                    : bucket_threshold([&](int i) { return vals[i]; }, n, kx, vmax, hist, &bs);
        if (ncand >= kx && ncand <= CAP) {
            // candidates go to their bucket's range; buckets are in value order
            bucket_starts(hist, cur);
            for (int i = lane; i < n; i += 32) {
                const float v = vals[i];
                if (bucket_of(vmax, v) <= bs) {
                    const uint32_t pos = atomicAdd(&cur[bucket_of(vmax, v)], 1u);
                    tmp[pos] = ((uint64_t)f2key(v) << 32) | (uint64_t)(0xffffffffu - (uint32_t)i);
                }
            }
            __syncwarp();
            // inside a bucket, order by (key desc, index asc): rank among its peers
            for (int pos = lane; pos < ncand; pos += 32) {
                const uint64_t k = tmp[pos];
                const int b = bucket_of(vmax, key2f((uint32_t)(k >> 32)));
                const int s0 = (int)hist[b];
                const int s1 = b < bs ? (int)hist[b + 1] : ncand;
                int r = 0;
                for (int q = s0; q < s1; ++q) r += tmp[q] > k ? 1 : 0;
                const int fp = s0 + r;
                if (fp < kx) {
                    oval[fp] = key2f((uint32_t)(k >> 32));
                    oidx[fp] = (int)(0xffffffffu - (uint32_t)k);
                }
            }
            return;
        }
    }

    // ---- exact fallback: radix select on keys, rank sort
    uint32_t *keys = reinterpret_cast<uint32_t *>(vals);
    for (int i = lane; i < n; i += 32) keys[i] = f2key(vals[i]);
    __syncwarp();
    int take_eq;
    const uint32_t T = warp_radix_select(keys, n, kx, hist, &take_eq);
    int taken = 0, eq_seen = 0;
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + (int)lane;
        const uint32_t key = i < n ? keys[i] : 0u;
        const bool gt = i < n && key > T;
        const bool eq = i < n && key == T;
        const unsigned beq = __ballot_sync(0xffffffffu, eq);
        const int eq_rank = eq_seen + __popc(beq & lanemask_lt());
        const bool take = gt || (eq && eq_rank < take_eq);
        const unsigned bt = __ballot_sync(0xffffffffu, take);
        if (take) {
            const int pos = taken + __popc(bt & lanemask_lt());
            sel_key[pos] = key;
            sel_idx[pos] = i;
        }
        taken += __popc(bt);
        eq_seen += __popc(beq);
    }
    __syncwarp();
    for (int u = lane; u < kx; u += 32) {
        const uint32_t ku = sel_key[u];
        int r = 0;
        for (int v = 0; v < kx; ++v) {
            const uint32_t kv = sel_key[v];
            r += (kv > ku) | ((kv == ku) & (v < u));
        }
        oval[r] = key2f(ku);
        oidx[r] = sel_idx[u];
    }
}

template <int CAP>
__global__ void axis_topk_kernel(const float *__restrict__ in_r, const float *__restrict__ in_c,
                                 int logsoftmax, const float2 *__restrict__ part_r,
                                 const float2 *__restrict__ part_c, float *__restrict__ p_r_out,
                                 float *__restrict__ p_c_out, int L, int N_r, int N_c, int K,
                                 float *__restrict__ row_val, int *__restrict__ row_idx,
                                 float *__restrict__ col_val, int *__restrict__ col_idx,
                                 int nmax, int kmax, size_t warp_words,
                                 const int *__restrict__ only) {
    extern __shared__ __align__(16) uint32_t smem_u[];
    grid_dependency_wait();
    grid_dependents_launch();
    const int warp = threadIdx.x >> 5;
    const int wpb = blockDim.x >> 5;
    const int64_t prob = (int64_t)blockIdx.x * wpb + warp;
    if (prob >= 2 * (int64_t)L) return;
    if (only && only[prob] == 0) return;          // handled by the register kernel
    const int t = (int)(prob >> 1);
    const int axis = (int)(prob & 1);
    const int n = axis ? N_c : N_r;
    const int kx = K < n ? K : n;
    axis_row_exact<CAP>((axis ? in_c : in_r) + (size_t)t * n, n, kx, logsoftmax,
                        axis ? part_c : part_r, t, axis ? p_c_out : p_r_out,
                        (axis ? col_val : row_val) + (size_t)t * kx,
                        (axis ? col_idx : row_idx) + (size_t)t * kx, nmax, kmax,
                        smem_u + (size_t)warp * warp_words);
}

// ------------------------------------------------- axis top-K, registers
// Fast path for rows with n % 4 == 0 and n <= 128 * NPL: lane l holds float4
// number l + 32 j of the row (j < NPL) in registers.  mode 0: the input is
// p; mode 1: p = s - lse with lse from the GEMM partials; mode 2: p = s - lse
// computed here.  A row the bucket sort cannot finish (too few values within
// 8 units of the maximum, or more than CAP candidates) is redone by the same
// warp with the exact radix select of axis_row_exact, which reads the row
// again.  Shared memory per warp (warp_words, even): hist[kNB] | cur[kNB] |
// tmp[CAP] (u64), or axis_row_exact's area for nmax, kmax.  Up to 11 float4
// per lane, at most 96 registers, so that five CTAs share an SM.
template <int NPL, int CAP>
__global__ void __launch_bounds__(128, NPL <= 11 ? 5 : 4)
axis_topk_reg_kernel(const float *__restrict__ in_r, const float *__restrict__ in_c, int mode,
                     const float2 *__restrict__ part_r, const float2 *__restrict__ part_c,
                     float *__restrict__ p_r_out, float *__restrict__ p_c_out, int L, int N_r,
                     int N_c, int K, float *__restrict__ row_val, int *__restrict__ row_idx,
                     float *__restrict__ col_val, int *__restrict__ col_idx, int nmax, int kmax,
                     int warp_words) {
    extern __shared__ __align__(16) uint32_t smem_u[];
    grid_dependency_wait();
    grid_dependents_launch();
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    const int64_t prob = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
    if (prob >= 2 * (int64_t)L) return;
    const int t = (int)(prob >> 1);
    const int axis = (int)(prob & 1);
    const int n = axis ? N_c : N_r;
    const int n4 = n >> 2;
    const int kx = K < n ? K : n;
    const float4 *in4 = reinterpret_cast<const float4 *>((axis ? in_c : in_r) + (size_t)t * n);
    float *pout = axis ? p_c_out : p_r_out;
    uint32_t *hist = smem_u + (size_t)warp * warp_words;
    uint32_t *cur = hist + kNB;
    uint64_t *tmp = reinterpret_cast<uint64_t *>(cur + kNB);

    float4 v[NPL];
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
        const int i4 = (int)lane + 32 * j;
        v[j] = i4 < n4 ? in4[i4] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    }
    float lse = 0.f, vmax;
    if (mode == 1) {
        float mx;
        lse = lse_from_partials(axis ? part_c : part_r, t, n, &mx);
        vmax = mx - lse;
    } else {
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < NPL; ++j)
            mx = fmaxf(fmaxf(mx, fmaxf(v[j].x, v[j].y)), fmaxf(v[j].z, v[j].w));
        mx = warp_max(mx);
        if (mode == 2) {
            float sum = 0.f;
#pragma unroll
            for (int j = 0; j < NPL; ++j)
                if ((int)lane + 32 * j < n4)
                    sum += __expf(v[j].x - mx) + __expf(v[j].y - mx) + __expf(v[j].z - mx) +
                           __expf(v[j].w - mx);
            sum = warp_sum(sum);
            lse = mx + __logf(sum);
            vmax = mx - lse;
        } else {
            vmax = mx;
        }
    }
    if (mode != 0) {
#pragma unroll
        for (int j = 0; j < NPL; ++j) {
            v[j].x -= lse;
            v[j].y -= lse;
            v[j].z -= lse;
            v[j].w -= lse;
        }
        if (pout) {
            float *prow = pout + (size_t)t * n;
            const bool vec = (reinterpret_cast<uintptr_t>(prow) & 15u) == 0;
#pragma unroll
            for (int j = 0; j < NPL; ++j) {
                const int i4 = (int)lane + 32 * j;
                if (i4 < n4) {
                    if (vec) {
                        reinterpret_cast<float4 *>(prow)[i4] = v[j];
                    } else {
                        prow[4 * i4] = v[j].x;
                        prow[4 * i4 + 1] = v[j].y;
                        prow[4 * i4 + 2] = v[j].z;
                        prow[4 * i4 + 3] = v[j].w;
                    }
                }
            }
        }
    }
    for (int b = lane; b < kNB; b += 32) hist[b] = 0u;
    __syncwarp();
    auto count = [&](float p) {
        const int b = bucket_of(vmax, p);
        if (b < kNB) atomicAdd(&hist[b], 1u);
    };
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
        count(v[j].x);
        count(v[j].y);
        count(v[j].z);
        count(v[j].w);
    }
    __syncwarp();
    int bs = 0;
    const int ncand = bucket_find(hist, kx, &bs);
    float *oval = (axis ? col_val : row_val) + (size_t)t * kx;
    int *oidx = (axis ? col_idx : row_idx) + (size_t)t * kx;
    if (ncand < kx || ncand > CAP) {
        __syncwarp();
        axis_row_exact<0>((axis ? in_c : in_r) + (size_t)t * n, n, kx, mode != 0,
                          mode == 1 ? (axis ? part_c : part_r) : nullptr, t, pout, oval, oidx,
                          nmax, kmax, hist);
        return;
    }
    bucket_starts(hist, cur);
    auto place = [&](float p, int i) {
        const int b = bucket_of(vmax, p);
        if (b <= bs) {
            const uint32_t pos = atomicAdd(&cur[b], 1u);
            tmp[pos] = ((uint64_t)f2key(p) << 32) | (uint64_t)(0xffffffffu - (uint32_t)i);
        }
    };
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
        const int i = 4 * ((int)lane + 32 * j);
        place(v[j].x, i);
        place(v[j].y, i + 1);
        place(v[j].z, i + 2);
        place(v[j].w, i + 3);
    }
    __syncwarp();
    for (int pos = lane; pos < ncand; pos += 32) {
        const uint64_t k = tmp[pos];
        const int b = bucket_of(vmax, key2f((uint32_t)(k >> 32)));
        const int s0 = (int)hist[b];
        const int s1 = b < bs ? (int)hist[b + 1] : ncand;
        int r = 0;
        for (int q = s0; q < s1; ++q) r += tmp[q] > k ? 1 : 0;
        const int fp = s0 + r;
        if (fp < kx) {
            oval[fp] = key2f((uint32_t)(k >> 32));
            oidx[fp] = (int)(0xffffffffu - (uint32_t)k);
        }
    }
}

// ----------------------------------------------------------- merge top-K
struct Cand {          // one grid cell of the candidate block
    uint32_t skey;     // key(S)
    uint32_t prkey;    // key(p_r[i])
    uint32_t pckey;    // key(p_c[j])
    uint32_t n;        // i * N_c + j
};

// true if cell u ranks before cell v
__device__ __forceinline__ bool better(const Cand &u, const Cand &v) {
    if (u.skey != v.skey) return u.skey > v.skey;
    if (u.prkey != v.prkey) return u.prkey > v.prkey;
    if (u.pckey != v.pckey) return u.pckey > v.pckey;
    return u.n < v.n;
}

struct MergeLayout {   // offsets (words) inside one warp's region
    size_t rv, ri, cv, ci, hist, q, out_s, out_n, words;
};

// Per warp: rv, ri [Kr], cv, ci [Kc] (the token's row and column top-K),
// hist [kNB] (bucket counts, then bucket starts, then bucket ends), the area
// q of max(4 CAP, C) words (the fast path's 128-bit candidate keys, or the
// fallback's candidate keys and then the indices it keeps), out_S, out_n [K].
__host__ __device__ inline MergeLayout merge_layout(int K, int Kr, int Kc, int C, int cap) {
    MergeLayout m;
    size_t o = 0;
    m.rv = o; o += Kr;
    m.ri = o; o += Kr;
    m.cv = o; o += Kc;
    m.ci = o; o += Kc;
    m.hist = o; o += kNB;
    o = (o + 3) & ~(size_t)3;                 // 16-byte alignment for the u64 keys
    m.q = o; o += (4 * (size_t)cap > (size_t)C ? 4 * (size_t)cap : (size_t)C);
    m.out_s = o; o += K;
    m.out_n = o; o += K;
    m.words = (o + 3) & ~(size_t)3;
    return m;
}

// Drops from L2, without a write-back, the 128-byte lines lying wholly
// inside [p, p + n) (discard.global.L2 leaves their contents undefined).
__device__ __forceinline__ void discard_l2_lines(const float *p, int n) {
    const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
    const uintptr_t first = (lo + 127u) & ~(uintptr_t)127u;
    const uintptr_t end = (lo + (uintptr_t)n * 4u) & ~(uintptr_t)127u;
    for (uintptr_t a = first + 128u * lane_id(); a < end; a += 128u * 32u)
        asm volatile("discard.global.L2 [%0], 128;" ::"l"(a) : "memory");
}

// Candidate table (the whole CTA): table[c] = (a << 16) | b for the c-th cell
// (a, b) with (a+1)(b+1) <= K, a-major; off (Kr + 1 ints) is scratch.
__device__ void merge_table(int K, int Kr, int Kc, int C, uint32_t *table, int *off) {
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    if (warp == 0) {
        int carry = 0;
        for (int a0 = 0; a0 < Kr; a0 += 32) {
            const int a = a0 + (int)lane;
            int nb = 0;
            if (a < Kr) {
                nb = K / (a + 1);
                if (nb > Kc) nb = Kc;
            }
            const int inc = warp_iscan(nb);
            if (a < Kr) off[a] = carry + inc - nb;
            carry += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) off[Kr] = carry;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        int lo = 0, hi = Kr - 1;                 // last a with off[a] <= c
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (off[mid] <= c) lo = mid; else hi = mid - 1;
        }
        table[c] = ((uint32_t)lo << 16) | (uint32_t)(c - off[lo]);
    }
    __syncthreads();

}

// One token, one warp: the global top-K of S = fl32(p_r[i] + p_c[j]) over the
// candidate cells from the token's row and column top-K (row_val / row_idx:
// Kr entries, col_val / col_idx: Kc entries), ranked by (S, p_r, p_c, n), and
// the gates; idx / score / gate are the token's K outputs.  `base` is the
// warp's shared area (merge_layout), `table` the CTA's candidate table.
template <int CAP>
__device__ void merge_token(const uint32_t *table, uint32_t *base, const MergeLayout &ml,
                            const float *__restrict__ row_val, const int *__restrict__ row_idx,
                            const float *__restrict__ col_val, const int *__restrict__ col_idx,
                            int N_c, int K, int Kr, int Kc, int C, int t, int32_t *idx,
                            float *score, float *gate, const SchedPrep &prep) {
    const unsigned lane = lane_id();
    float *rv = reinterpret_cast<float *>(base + ml.rv);
    uint32_t *ri = base + ml.ri;
    float *cv = reinterpret_cast<float *>(base + ml.cv);
    uint32_t *ci = base + ml.ci;
    uint32_t *hist = base + ml.hist;
    uint32_t *qw = base + ml.q;
    uint64_t *tmp = reinterpret_cast<uint64_t *>(base + ml.q);
    float *out_S = reinterpret_cast<float *>(base + ml.out_s);
    uint32_t *out_n = base + ml.out_n;

    for (int a = lane; a < Kr; a += 32) {
        rv[a] = row_val[a];
        ri[a] = (uint32_t)row_idx[a];
    }
    for (int b = lane; b < Kc; b += 32) {
        cv[b] = col_val[b];
        ci[b] = (uint32_t)col_idx[b];
    }
    __syncwarp();
    const float smax = __fadd_rn(rv[0], cv[0]);           // cell (0, 0) is the largest
    // S of candidate c (one fp32 addition, recomputed where needed)
    auto score_of = [&](int c, int *a_out, int *b_out) {
        const uint32_t ab = table[c];
        *a_out = (int)(ab >> 16);
        *b_out = (int)(ab & 0xffffu);
        return __fadd_rn(rv[*a_out], cv[*b_out]);
    };

    bool done = false;
    if (CAP > 0) {
        for (int b = lane; b < kNB; b += 32) hist[b] = 0u;
        __syncwarp();
        for (int c = lane; c < C; c += 32) {
            int a, b2;
            const int b = bucket_of(smax, score_of(c, &a, &b2));
            if (b < kNB) atomicAdd(&hist[b], 1u);
        }
        __syncwarp();
        int bs = 0;
        const int ncand = bucket_find(hist, K, &bs);
        if (ncand >= K && ncand <= CAP) {
            // counts -> bucket starts, in place; the scatter below advances
            // each bucket's entry to its end
            {
                constexpr int per = kNB / 32;
                uint32_t cnt[per];
                int tot = 0;
#pragma unroll
                for (int j = 0; j < per; ++j) {
                    cnt[j] = hist[lane * per + j];
                    tot += (int)cnt[j];
                }
                int run = warp_iscan(tot) - tot;
#pragma unroll
                for (int j = 0; j < per; ++j) {
                    hist[lane * per + j] = (uint32_t)run;
                    run += (int)cnt[j];
                }
                __syncwarp();
            }
            for (int c = lane; c < C; c += 32) {
                int a, bb;
                const float S = score_of(c, &a, &bb);
                const int b = bucket_of(smax, S);
                if (b <= bs) {
                    const uint32_t pos = atomicAdd(&hist[b], 1u);
                    const uint32_t nn = ri[a] * (uint32_t)N_c + ci[bb];
                    tmp[2 * pos] = ((uint64_t)f2key(S) << 32) | f2key(rv[a]);
                    tmp[2 * pos + 1] = ((uint64_t)f2key(cv[bb]) << 32) | (uint64_t)(0xffffffffu - nn);
                }
            }
            __syncwarp();
            // inside a bucket, order by the full key: rank among its peers
            // (bucket b now spans [end of b - 1, end of b))
            for (int pos = lane; pos < ncand; pos += 32) {
                const uint64_t kh = tmp[2 * pos], kl = tmp[2 * pos + 1];
                const int b = bucket_of(smax, key2f((uint32_t)(kh >> 32)));
                const int s0 = b > 0 ? (int)hist[b - 1] : 0;
                const int s1 = (int)hist[b];
                int r = 0;
                for (int q = s0; q < s1; ++q) {
                    const uint64_t qh = tmp[2 * q], ql = tmp[2 * q + 1];
                    r += (qh > kh || (qh == kh && ql > kl)) ? 1 : 0;
                }
                const int fp = s0 + r;
                if (fp < K) {
                    out_S[fp] = key2f((uint32_t)(kh >> 32));
                    out_n[fp] = 0xffffffffu - (uint32_t)kl;
                }
            }
            done = true;
        }
    }
    if (!done) {
        // ---- exact fallback: radix select on key(S), then a rank sort by the
        // full key of the kept candidates (their keys recomputed from the
        // candidate table, so only their indices are stored)
        uint32_t *ckey = qw;
        for (int c = lane; c < C; c += 32) {
            int a, b;
            ckey[c] = f2key(score_of(c, &a, &b));
        }
        __syncwarp();
        int take_eq;
        const uint32_t T = warp_radix_select(ckey, C, K, hist, &take_eq);
        // keep the candidates with key >= T, compacted in place (a round reads
        // its 32 keys before any write, and writes only below them)
        int nq = 0;
        for (int c0 = 0; c0 < C; c0 += 32) {
            const int c = c0 + (int)lane;
            const bool in_q = c < C && ckey[c] >= T;
            const unsigned bal = __ballot_sync(0xffffffffu, in_q);
            __syncwarp();
            if (in_q) qw[nq + __popc(bal & lanemask_lt())] = (uint32_t)c;
            nq += __popc(bal);
            __syncwarp();
        }
        auto cand_of = [&](int c) {
            int a, b;
            const float S = score_of(c, &a, &b);
            Cand cd;
            cd.skey = f2key(S);
            cd.prkey = f2key(rv[a]);
            cd.pckey = f2key(cv[b]);
            cd.n = ri[a] * (uint32_t)N_c + ci[b];
            return cd;
        };
        for (int u = lane; u < nq; u += 32) {
            const Cand cu = cand_of((int)qw[u]);
            int r = 0;
            for (int v = 0; v < nq; ++v) r += better(cand_of((int)qw[v]), cu) ? 1 : 0;
            if (r < K) {
                out_S[r] = key2f(cu.skey);
                out_n[r] = cu.n;
            }
        }
    }
    __syncwarp();
    // gates: softmax over the K selected S (S sorted, out_S[0] is the max)
    const float smx = out_S[0];
    float part = 0.f;
    for (int k = lane; k < K; k += 32) part += expf(out_S[k] - smx);
    const float den = warp_sum(part);
    for (int k = lane; k < K; k += 32) {
        const float S = out_S[k];
        const float g = expf(S - smx) / den;
        idx[k] = (int32_t)out_n[k];
        score[k] = S;
        gate[k] = g;
        out_S[k] = g;                                 // this lane's entries only
    }
    if (prep.a_tok) {
        // the schedule's per-token step on the selection still on chip
        __syncwarp();
        sched_token(prep, t, K, reinterpret_cast<const int32_t *>(out_n),
                    [&](int u) { return out_S[u]; });
    }
}

// dead_r / dead_c (may be null): the router GEMM's logits s_r [L, N_r] and
// s_c [L, N_c] in the library's workspace.  Every reader of them has finished
// when this kernel runs, so each warp drops its token's rows from L2: about
// 43 MB of dirty lines at 4096 tokens of 2 x 1304 logits that would otherwise
// be written back to HBM while the expert stage streams its rows.
template <int CAP>
__global__ void merge_topk_kernel(const float *__restrict__ row_val,
                                  const int *__restrict__ row_idx,
                                  const float *__restrict__ col_val,
                                  const int *__restrict__ col_idx, int L, int N_c, int K, int Kr,
                                  int Kc, int C, int32_t *__restrict__ idx,
                                  float *__restrict__ score, float *__restrict__ gate,
                                  const float *dead_r, const float *dead_c, int N_r,
                                  SchedPrep prep) {
    extern __shared__ __align__(16) uint32_t smem_u[];
    grid_dependency_wait();
    grid_dependents_launch();
    const int warp = threadIdx.x >> 5;
    const int wpb = blockDim.x >> 5;
    const MergeLayout ml = merge_layout(K, Kr, Kc, C, CAP);
    uint32_t *table = smem_u;                                   // C entries
    int *off = reinterpret_cast<int *>(table + C);               // Kr + 1 entries
    const size_t head = ((size_t)C + Kr + 1 + 3) & ~(size_t)3;
    merge_table(K, Kr, Kc, C, table, off);
    const int t = blockIdx.x * wpb + warp;
    if (t >= L) return;
    if (dead_r) {
        discard_l2_lines(dead_r + (size_t)t * N_r, N_r);
        discard_l2_lines(dead_c + (size_t)t * N_c, N_c);
    }
    merge_token<CAP>(table, smem_u + head + (size_t)warp * ml.words, ml,
                     row_val + (size_t)t * Kr, row_idx + (size_t)t * Kr,
                     col_val + (size_t)t * Kc, col_idx + (size_t)t * Kc, N_c, K, Kr, Kc, C, t,
                     idx + (size_t)t * K, score + (size_t)t * K, gate + (size_t)t * K, prep);
}

// candidates the fast path takes (the k best plus the boundary bucket); 0 = none
int fast_capacity(int k) {
    return k <= 1024 ? ((k + 64 + 31) / 32) * 32 : 0;
}

// ------------------------------------------------ block-wide exact selection
// Used by the fused decode step, where one token's selection is on the
// critical path: many threads per row instead of one warp.

// Named barrier over `nthreads` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Exact radix select of the k largest of the 32-bit keys key(i), i < n, by
// `nt` threads (thread ht of them, ht < nt) sharing `hist` (kNB words) and
// `scr` (2 words).  Returns T, the k-th largest key, and sets *take_eq to how
// many keys equal to T belong to the k largest (every key > T does).
template <typename KeyOf>
__device__ uint32_t group_radix_select(KeyOf key_of, int n, int k, int ht, int nt, int bar_id,
                                       uint32_t *hist, int *scr, int *take_eq) {
    uint32_t prefix = 0, mask = 0;
    int krem = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = ht; b < kNB; b += nt) hist[b] = 0u;
        named_sync(bar_id, nt);
        // keys that share the prefix crowd a few digits (all log-probabilities
        // share the top byte): lanes with the same digit add with one atomic
        for (int i0 = 0; i0 < n; i0 += nt) {
            const int i = i0 + ht;
            uint32_t dg = kNB;                                   // no digit
            if (i < n) {
                const uint32_t key = key_of(i);
                if ((key & mask) == prefix) dg = (key >> shift) & 255u;
            }
            const unsigned peers = __match_any_sync(0xffffffffu, dg);
            if (dg < (uint32_t)kNB && lane_id() == (unsigned)(__ffs(peers) - 1))
                atomicAdd(&hist[dg], (uint32_t)__popc(peers));
        }
        named_sync(bar_id, nt);
        if (ht < 32) {
            // lane l owns bins 255-8l down to 248-8l (largest digits first)
            int c[8], tot = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = (int)hist[255 - 8 * ht - j];
                tot += c[j];
            }
            const int incl = warp_iscan(tot);
            const int excl = incl - tot;
            const bool mine = excl < krem && krem <= incl;
            if (mine) {
                int run = excl;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (run + c[j] >= krem) {
                        scr[0] = 255 - 8 * ht - j;
                        scr[1] = run;
                        break;
                    }
                    run += c[j];
                }
            }
        }
        named_sync(bar_id, nt);
        const int digit = scr[0], above = scr[1];
        krem -= above;
        prefix |= (uint32_t)digit << shift;
        mask |= 255u << shift;
        named_sync(bar_id, nt);                      // scr is rewritten by the next pass
    }
    *take_eq = krem;
    return prefix;
}

// Sum / max of one float per thread over nt threads (warp-level, then
// through `red` (nt / 32 floats)).
__device__ __forceinline__ float group_sum(float v, int ht, int nt, int bar_id, float *red) {
    v = warp_sum(v);
    if ((ht & 31) == 0) red[ht >> 5] = v;
    named_sync(bar_id, nt);
    float t = 0.f;
    for (int w = 0; w < nt / 32; ++w) t += red[w];
    named_sync(bar_id, nt);
    return t;
}
__device__ __forceinline__ float group_max(float v, int ht, int nt, int bar_id, float *red) {
    v = warp_max(v);
    if ((ht & 31) == 0) red[ht >> 5] = v;
    named_sync(bar_id, nt);
    float t = -INFINITY;
    for (int w = 0; w < nt / 32; ++w) t = fmaxf(t, red[w]);
    named_sync(bar_id, nt);
    return t;
}

// One (token, axis) row by nt threads: p = s - logsumexp(s), and the kx best
// by (p desc, index asc) into oval / oidx in that order.  The block-wide
// form of the warp's bucket counting sort: p is counted into value buckets
// below the row maximum, the bucket b* that holds the kx-th value is found,
// the candidates (buckets <= b*) are scattered to their bucket's range and
// each is ranked among its bucket peers only.  When more than tmp_cap values
// fall in those buckets (or fewer than kx in range), an exact radix select
// takes over.  Shared: vals (n words), hist, cur (kNB each), tmp
// (max(tmp_cap, kx) 64-bit keys), scr (8 words).
// The exact selection of group_axis_select from the keys of p (in vals as
// raw words): radix select, ties by the smaller index, compaction and a rank
// sort into oval / oidx.
__device__ void group_axis_exact_keys(int n, int kx, int ht, int nt, int bar_id, float *vals,
                                      uint32_t *hist, uint64_t *tmp, int *scr, float *oval,
                                      int *oidx) {
    float *red = reinterpret_cast<float *>(scr + 2);
    auto key_of = [&](int i) { return __float_as_uint(vals[i]); };
    int take_eq;
    const uint32_t T = group_radix_select(key_of, n, kx, ht, nt, bar_id, hist, scr, &take_eq);
    // keys equal to T: the take_eq smallest indices (by radix select on the
    // inverted index among them, when there are more)
    int n_eq = 0;
    for (int i = ht; i < n; i += nt) n_eq += key_of(i) == T ? 1 : 0;
    n_eq = (int)group_sum((float)n_eq, ht, nt, bar_id, red);
    uint32_t Tl = 0u;
    if (n_eq > take_eq) {
        int tl_eq;
        Tl = group_radix_select([&](int i) { return key_of(i) == T ? 0xffffffffu - (uint32_t)i : 0u; },
                                n, take_eq, ht, nt, bar_id, hist, scr, &tl_eq);
    }
    // compact the kx selected (64-bit keys: p key, inverted index), one
    // atomic per warp and round
    if (ht == 0) scr[0] = 0;
    named_sync(bar_id, nt);
    for (int i0 = 0; i0 < n; i0 += nt) {
        const int i = i0 + ht;
        bool take = false;
        uint32_t key = 0u, lo = 0u;
        if (i < n) {
            key = key_of(i);
            lo = 0xffffffffu - (uint32_t)i;
            take = key > T || (key == T && (n_eq == take_eq || lo >= Tl));
        }
        const unsigned bal = __ballot_sync(0xffffffffu, take);
        int base = 0;
        if (bal && lane_id() == 0) base = atomicAdd(&scr[0], __popc(bal));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (take) {
            const int at = base + __popc(bal & lanemask_lt());
            if (at < kx) tmp[at] = ((uint64_t)key << 32) | lo;
        }
    }
    named_sync(bar_id, nt);
    // rank sort (keys are distinct)
    for (int j = ht; j < kx; j += nt) {
        const uint64_t kj = tmp[j];
        int r = 0;
        for (int i = 0; i < kx; ++i) r += tmp[i] > kj;
        oval[r] = key2f((uint32_t)(kj >> 32));
        oidx[r] = (int)(0xffffffffu - (uint32_t)kj);
    }
    named_sync(bar_id, nt);
}

// (m, s) pairs of a running logsumexp: s = sum exp(v - m) over the values
// seen; m = -inf with s = 0 for none.
__device__ __forceinline__ void lse_combine(float &m, float &s, float m2, float s2) {
    const float mx = fmaxf(m, m2);
    if (mx == -INFINITY) return;
    s = (m == -INFINITY ? 0.f : s * __expf(m - mx)) + (m2 == -INFINITY ? 0.f : s2 * __expf(m2 - mx));
    m = mx;
}

constexpr int kAxisRegJ = 4;    // float4 per thread held in registers by group_axis_select

__device__ void group_axis_select(const float *__restrict__ in, int n, int kx, int ht, int nt,
                                  int bar_id, float *vals, uint32_t *hist, uint32_t *cur,
                                  uint64_t *tmp, int tmp_cap, int *scr, float *oval, int *oidx) {
    float *red = reinterpret_cast<float *>(scr + 2);
    for (int b = ht; b < kNB; b += nt) hist[b] = 0u;
    const int n4 = n >> 2;
    if ((n & 3) == 0 && (reinterpret_cast<uintptr_t>(in) & 15u) == 0 && n4 <= kAxisRegJ * nt) {
        // ---- the row in registers: one (max, sum exp) reduction, then the
        // bucket counts, the scatter and the rank without shared-memory passes
        const float4 *in4 = reinterpret_cast<const float4 *>(in);
        float4 v[kAxisRegJ];
#pragma unroll
        for (int j = 0; j < kAxisRegJ; ++j) {
            const int i4 = ht + j * nt;
            v[j] = i4 < n4 ? in4[i4] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        }
        float m = -INFINITY, sm_ = 0.f;
#pragma unroll
        for (int j = 0; j < kAxisRegJ; ++j)
            m = fmaxf(fmaxf(m, fmaxf(v[j].x, v[j].y)), fmaxf(v[j].z, v[j].w));
        if (m > -INFINITY) {
#pragma unroll
            for (int j = 0; j < kAxisRegJ; ++j)
                sm_ += __expf(v[j].x - m) + __expf(v[j].y - m) + __expf(v[j].z - m) + __expf(v[j].w - m);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, sm_, o);
            lse_combine(m, sm_, m2, s2);
        }
        float2 *red2 = reinterpret_cast<float2 *>(tmp);          // nt / 32 pairs, before tmp is used
        if ((ht & 31) == 0) red2[ht >> 5] = make_float2(m, sm_);
        named_sync(bar_id, nt);
        float M = -INFINITY, S = 0.f;
        for (int w = 0; w < nt / 32; ++w) lse_combine(M, S, red2[w].x, red2[w].y);
        const float lse = M + __logf(S);
        const float vmax = M - lse;                 // the p of the largest logit, same rounding
#pragma unroll
        for (int j = 0; j < kAxisRegJ; ++j) {
            v[j].x -= lse; v[j].y -= lse; v[j].z -= lse; v[j].w -= lse;
            if (ht + j * nt < n4) {
                const float q[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int b = bucket_of(vmax, q[c]);
                    if (b < kNB) atomicAdd(&hist[b], 1u);
                }
            }
        }
        named_sync(bar_id, nt);                     // counts complete; red2 no longer read
        if (ht < 32) {
            int bs = 0;
            const int nc = bucket_scan(hist, cur, kx, &bs);
            if (ht == 0) {
                scr[0] = nc >= kx && nc <= tmp_cap ? nc : -1;
                scr[1] = bs;
            }
        }
        named_sync(bar_id, nt);
        const int ncand = scr[0], bstar = scr[1];
        if (ncand >= 0) {
#pragma unroll
            for (int j = 0; j < kAxisRegJ; ++j) {
                if (ht + j * nt < n4) {
                    const float q[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int b = bucket_of(vmax, q[c]);
                        if (b <= bstar) {
                            const int i = 4 * (ht + j * nt) + c;
                            tmp[atomicAdd(&cur[b], 1u)] =
                                ((uint64_t)f2key(q[c]) << 32) | (uint64_t)(0xffffffffu - (uint32_t)i);
                        }
                    }
                }
            }
            named_sync(bar_id, nt);
            for (int pos = ht; pos < ncand; pos += nt) {
                const uint64_t k = tmp[pos];
                const float p = key2f((uint32_t)(k >> 32));
                const int b = bucket_of(vmax, p);
                const int s0 = (int)hist[b], s1 = b < bstar ? (int)hist[b + 1] : ncand;
                int r = 0;
                for (int q = s0; q < s1; ++q) r += tmp[q] > k ? 1 : 0;
                if (s0 + r < kx) {
                    oval[s0 + r] = p;
                    oidx[s0 + r] = (int)(0xffffffffu - (uint32_t)k);
                }
            }
            named_sync(bar_id, nt);
            return;
        }
        // the exact fallback below starts from the keys of p in shared memory
#pragma unroll
        for (int j = 0; j < kAxisRegJ; ++j) {
            const int i4 = ht + j * nt;
            if (i4 < n4)
                reinterpret_cast<float4 *>(vals)[i4] =
                    make_float4(__uint_as_float(f2key(v[j].x)), __uint_as_float(f2key(v[j].y)),
                                __uint_as_float(f2key(v[j].z)), __uint_as_float(f2key(v[j].w)));
        }
        named_sync(bar_id, nt);
        group_axis_exact_keys(n, kx, ht, nt, bar_id, vals, hist, tmp, scr, oval, oidx);
        return;
    }
    // the row with every load in flight, its maximum
    float mx = -INFINITY;
    if ((n & 3) == 0 && (reinterpret_cast<uintptr_t>(in) & 15u) == 0) {
        const float4 *in4 = reinterpret_cast<const float4 *>(in);
        float4 *v4 = reinterpret_cast<float4 *>(vals);
#pragma unroll 4
        for (int i4 = ht; i4 < (n >> 2); i4 += nt) {
            const float4 v = in4[i4];
            v4[i4] = v;
            mx = fmaxf(fmaxf(mx, fmaxf(v.x, v.y)), fmaxf(v.z, v.w));
        }
    } else {
#pragma unroll 4
        for (int i = ht; i < n; i += nt) {
            const float v = in[i];
            vals[i] = v;
            mx = fmaxf(mx, v);
        }
    }
    mx = group_max(mx, ht, nt, bar_id, red);
    float sm_ = 0.f;
    for (int i = ht; i < n; i += nt) sm_ += __expf(vals[i] - mx);
    const float lse = mx + __logf(group_sum(sm_, ht, nt, bar_id, red));
    const float vmax = mx - lse;                 // the p of the largest logit, same rounding
    for (int i = ht; i < n; i += nt) {
        const float p = vals[i] - lse;
        vals[i] = p;
        const int b = bucket_of(vmax, p);
        if (b < kNB) atomicAdd(&hist[b], 1u);
    }
    named_sync(bar_id, nt);
    if (ht < 32) {                               // the group's first warp
        int bs = 0;
        const int nc = bucket_scan(hist, cur, kx, &bs);
        const bool fast = nc >= kx && nc <= tmp_cap;
        if (ht == 0) {
            scr[0] = fast ? nc : -1;
            scr[1] = bs;
        }
    }
    named_sync(bar_id, nt);
    const int ncand = scr[0], bstar = scr[1];
    if (ncand >= 0) {
        for (int i = ht; i < n; i += nt) {
            const float p = vals[i];
            const int b = bucket_of(vmax, p);
            if (b <= bstar)
                tmp[atomicAdd(&cur[b], 1u)] =
                    ((uint64_t)f2key(p) << 32) | (uint64_t)(0xffffffffu - (uint32_t)i);
        }
        named_sync(bar_id, nt);
        for (int pos = ht; pos < ncand; pos += nt) {
            const uint64_t k = tmp[pos];
            const float p = key2f((uint32_t)(k >> 32));
            const int b = bucket_of(vmax, p);
            const int s0 = (int)hist[b], s1 = b < bstar ? (int)hist[b + 1] : ncand;
            int r = 0;
            for (int q = s0; q < s1; ++q) r += tmp[q] > k ? 1 : 0;
            if (s0 + r < kx) {
                oval[s0 + r] = p;
                oidx[s0 + r] = (int)(0xffffffffu - (uint32_t)k);
            }
        }
        named_sync(bar_id, nt);
        return;
    }

    // ---- exact fallback: radix select on the keys of p
    for (int i = ht; i < n; i += nt) vals[i] = __uint_as_float(f2key(vals[i]));
    named_sync(bar_id, nt);
    group_axis_exact_keys(n, kx, ht, nt, bar_id, vals, hist, tmp, scr, oval, oidx);
}

// Shared words of the block-wide merge (group_merge) ahead of its candidate
// keys: hist, cur, the dense ranks of the row and column lists (128 each),
// 16 words of scratch, out_S and out_n (K each); even, so that the 64-bit
// keys that follow are aligned.
__host__ __device__ inline int group_merge_head_words(int K) {
    return (2 * kNB + 256 + 16 + 2 * K + 1) & ~1;
}

// The merge of one token by the whole CTA (256 threads): the global top-K of
// S = fl32(p_r[a] + p_c[b]) over the candidate cells (a, b) of `table`,
// ranked by (S desc, p_r desc, p_c desc, n asc), and the gates.  Kr, Kc <=
// 128.  Every cell gets one unique 64-bit key that encodes the whole rule:
// the key of S, then (dr[a], dc[b], a, b) ascending, where dr / dc are the
// dense ranks of the row / column list (equal p share a rank; the lists are
// in (p desc, index asc) order, so among equal p a smaller list position is
// a smaller index, and (a, b) ascending is n ascending).  The K largest keys
// are found by the bucket counting sort on S below S(0, 0) (every cell
// ranked among its bucket peers), or, when fewer than K cells are in range,
// by ranking every cell against all C.  rv / ri, cv / ci: the token's row and
// column top-K (shared); `work`: group_merge_head_words(K) + 2 C words.
__device__ void group_merge(const uint32_t *table, const float *rv, const int *ri, const float *cv,
                            const int *ci, int N_c, int K, int Kr, int Kc, int C, uint32_t *work,
                            int32_t *idx, float *score, float *gate) {
    const int ht = threadIdx.x, nt = blockDim.x;
    const unsigned lane = lane_id();
    const int warp = ht >> 5;
    uint32_t *hist = work, *cur = work + kNB;
    uint32_t *dr = cur + kNB, *dc = dr + 128;
    int *scr = reinterpret_cast<int *>(dc + 128);
    float *out_S = reinterpret_cast<float *>(scr + 16);
    uint32_t *out_n = reinterpret_cast<uint32_t *>(out_S + K);
    uint64_t *ckey = reinterpret_cast<uint64_t *>(work + group_merge_head_words(K));

    for (int b = ht; b < kNB; b += nt) hist[b] = 0u;
    // dense ranks: warps 0-3 the row list, warps 4-7 the column list
    const bool colw = ht >= 128;
    const int pos = ht & 127;
    const int nl = colw ? Kc : Kr;
    const float *lv = colw ? cv : rv;
    const bool flag = pos > 0 && pos < nl && f2key(lv[pos]) != f2key(lv[pos - 1]);
    const unsigned bal = __ballot_sync(0xffffffffu, flag);
    if (lane == 0) scr[warp] = __popc(bal);
    const float smax = __fadd_rn(rv[0], cv[0]);          // cell (0, 0) is the largest
    __syncthreads();
    {
        int before = 0;
        for (int w = colw ? 4 : 0; w < warp; ++w) before += scr[w];
        if (pos < nl) (colw ? dc : dr)[pos] = (uint32_t)(before + __popc(bal & lanemask_lt()) + (flag ? 1 : 0));
    }
    for (int c = ht; c < C; c += nt) {
        const uint32_t ab = table[c];
        const int b = bucket_of(smax, __fadd_rn(rv[ab >> 16], cv[ab & 0xffffu]));
        if (b < kNB) atomicAdd(&hist[b], 1u);
    }
    __syncthreads();
    if (ht < 32) {
        int bs = 0;
        const int nc = bucket_scan(hist, cur, K, &bs);
        const bool fast = nc >= K;
        if (ht == 0) {
            scr[8] = fast ? nc : -1;
            scr[9] = bs;
        }
    }
    __syncthreads();
    const int ncand = scr[8], bstar = scr[9];
    auto key_of = [&](uint32_t ab, float S) {
        const uint32_t a = ab >> 16, b = ab & 0xffffu;
        const uint32_t sec = (dr[a] << 24) | (dc[b] << 16) | (a << 8) | b;
        return ((uint64_t)f2key(S) << 32) | (uint64_t)(0xffffffffu - sec);
    };
    auto emit = [&](int at, uint64_t k) {
        const uint32_t sec = 0xffffffffu - (uint32_t)k;
        out_S[at] = key2f((uint32_t)(k >> 32));
        out_n[at] = (uint32_t)ri[(sec >> 8) & 255u] * (uint32_t)N_c + (uint32_t)ci[sec & 255u];
    };
    if (ncand >= 0) {
        for (int c = ht; c < C; c += nt) {
            const uint32_t ab = table[c];
            const float S = __fadd_rn(rv[ab >> 16], cv[ab & 0xffffu]);
            const int b = bucket_of(smax, S);
            if (b <= bstar) ckey[atomicAdd(&cur[b], 1u)] = key_of(ab, S);
        }
        __syncthreads();
        for (int j = ht; j < ncand; j += nt) {
            const uint64_t k = ckey[j];
            const int b = bucket_of(smax, key2f((uint32_t)(k >> 32)));
            const int s0 = (int)hist[b], s1 = b < bstar ? (int)hist[b + 1] : ncand;
            int r = 0;
            for (int q = s0; q < s1; ++q) r += ckey[q] > k ? 1 : 0;
            if (s0 + r < K) emit(s0 + r, k);
        }
    } else {
        for (int c = ht; c < C; c += nt) {
            const uint32_t ab = table[c];
            ckey[c] = key_of(ab, __fadd_rn(rv[ab >> 16], cv[ab & 0xffffu]));
        }
        __syncthreads();
        for (int j = ht; j < C; j += nt) {
            const uint64_t k = ckey[j];
            int r = 0;
            for (int q = 0; q < C; ++q) r += ckey[q] > k ? 1 : 0;
            if (r < K) emit(r, k);
        }
    }
    __syncthreads();
    // gates: softmax over the K selected S (out_S[0] is the max)
    if (ht < 32) {
        const float smx = out_S[0];
        float part = 0.f;
        for (int k = ht; k < K; k += 32) part += expf(out_S[k] - smx);
        const float den = warp_sum(part);
        for (int k = ht; k < K; k += 32) {
            const float S = out_S[k];
            idx[k] = (int32_t)out_n[k];
            score[k] = S;
            gate[k] = expf(S - smx) / den;
        }
    }
}

// ------------------------------------------------------- fused decode step
// For a handful of tokens the routed forward is latency-bound: six dependent
// launches, each starting cold, cost about 34 us at L = 1 against a 1.7 us
// roofline.  Tokens are independent once the router projection is done, so
// one cooperative launch (every CTA resident) runs the whole step in three
// phases separated by a grid barrier (a bounded wait):
//   A. the first gridDim.x - L CTAs: the router projection of their block
//      of router rows, pulled with the token rows into shared memory by
//      bulk copies (CUDA-core dot products for 1-2 tokens, mma.sync for
//      3-16) into s; y zeroed unless accumulating; the last L CTAs build the
//      merge's candidate table;
//   B. CTA gridDim.x - 1 - t, token t: LogSoftmax and the exact row and
//      column top-K (128 threads per axis, group_axis_select), then the
//      merge and the gates (the whole CTA, group_merge), with the ranking
//      rule of the separate kernels;
//   C. chunks of up to 8 tasks of one token per CTA: h = x_t . w_e,
//      p = g SiLU(h) per warp, the chunk's sum of p v_e per CTA, added to
//      y_t with 16-byte fp32 reductions (the order in which a token's chunks
//      land varies from run to run).
constexpr int kDecodeWarps = 8;
constexpr int kDecodeSlices = 8;           // 8-wide slices per lane: d <= 2048

struct DecodeArgs {
    const uint16_t *x, *W, *V, *W_r, *W_c;
    int L, d, N_r, N_c, K, Kr, Kc, C;
    int64_t N;
    float *s_r, *s_c;
    float *row_val, *col_val;
    int *row_idx, *col_idx;
    int32_t *idx;
    float *score, *gate;
    float *y;
    int accumulate;
    unsigned long long *bar;               // grid barrier: (epoch << 32) | arrivals
    unsigned epoch;                        // this call's tag, never 0, differs from the last call's
    int rpc;                               // router rows per projecting CTA
    int nproj;                             // projecting CTAs (the first ones)
    int *status;
    int nmax, kmax;
    int axis_words;                        // shared words per axis warp
    int merge_head;                        // candidate table and its scratch
    int list_words;                        // the token's row and column top-K (values, indices)
    int nmax_pad;                          // nmax rounded up to an even word count
    int tmp_cap;                           // candidates of the axis bucket sort
};

// All CTAs of the grid arrive; the wait gives up after kWaitLimitNs and
// records OMNI_DEV_WAIT_TIMEOUT (then the CTA returns).  The barrier word
// holds (epoch << 32) | arrivals and needs no clearing between calls: CTA 0
// installs (epoch, 0) with one exchange when the kernel starts, and an
// arrival that finds another call's epoch (it came before the exchange,
// which erased it) arrives again once the epoch is there.  Barrier k of the
// call completes at k * gridDim.x arrivals.
__device__ bool decode_grid_barrier(unsigned long long *bar, unsigned epoch, unsigned target,
                                    int *status, int *s_ok) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        bool counted = (unsigned)(atomicAdd(bar, 1ull) >> 32) == epoch;
        bool ok = true;
        const uint64_t t0 = global_timer_ns();
        // relaxed polls with a short back-off, one acquire fence at the end
        for (uint32_t it = 0;; ++it) {
            unsigned long long w;
            asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(bar) : "memory");
            if ((unsigned)(w >> 32) == epoch) {
                if (!counted) {
                    counted = (unsigned)(atomicAdd(bar, 1ull) >> 32) == epoch;
                    continue;
                }
                if ((unsigned)w >= target) {
                    asm volatile("fence.acq_rel.gpu;" ::: "memory");
                    break;
                }
            }
            if ((it & 63u) == 63u &&
                (it > kWaitSpinLimit || global_timer_ns() - t0 > kWaitLimitNs)) {
                set_status(status, OMNI_DEV_WAIT_TIMEOUT);
                ok = false;
                break;
            }
            __nanosleep(32);
        }
        *s_ok = ok ? 1 : 0;
    }
    __syncthreads();
    return *s_ok != 0;
}

// One 1-D bulk copy global -> this CTA's shared memory, completing on `bar`
// (16-byte aligned addresses, a multiple of 16 bytes).
__device__ __forceinline__ void bulk_load_1d(void *dst, const void *src, uint32_t bytes,
                                             uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// The projection of the CTA's nrow staged router rows with L staged token
// rows on the tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate):
// 16-row tiles of the block by 8-token tiles, the K = d loop split over the
// CTA's 8 warps, the warps' partial tiles summed through `red` (8 x 16 x 16
// floats of shared memory).  Rows and tokens past the end read the last
// staged one and their results are dropped.  A 10-row block is far below
// the 64-row minimum of a tcgen05 tile, and the warp-level instruction keeps
// the code short, which matters for a kernel fetched cold once per step.
__device__ void decode_rows_mma(const uint16_t *xs, const uint16_t *wsm, int nrow, int g0,
                                float *red, const DecodeArgs &a) {
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    const int kw = a.d / kDecodeWarps;                       // this warp's K range
    const int k_lo = warp * kw;
    const int ntile = (a.L + 7) >> 3;
    for (int m0 = 0; m0 < nrow; m0 += 16) {
        float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        // ldmatrix row addresses: A rows m0 + (lane % 16), B tokens lane % 8
        const int ar = min(m0 + (int)(lane & 15u), nrow - 1);
        const uint32_t a_base = smem_u32(wsm + (size_t)ar * a.d + k_lo + ((lane >> 4) << 3));
        uint32_t b_base[2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int bt = min(nt * 8 + (int)(lane & 7u), a.L - 1);
            b_base[nt] = smem_u32(xs + (size_t)bt * a.d + k_lo + (((lane >> 3) & 1u) << 3));
        }
#pragma unroll 4
        for (int k = 0; k < kw; k += 16) {
            uint32_t fa[4];
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                         : "=r"(fa[0]), "=r"(fa[1]), "=r"(fa[2]), "=r"(fa[3])
                         : "r"(a_base + 2u * k));
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                if (nt < ntile) {
                    uint32_t fb[2];
                    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
                                 : "=r"(fb[0]), "=r"(fb[1]) : "r"(b_base[nt] + 2u * k));
                    asm volatile(
                        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
                        : "+f"(c[nt][0]), "+f"(c[nt][1]), "+f"(c[nt][2]), "+f"(c[nt][3])
                        : "r"(fa[0]), "r"(fa[1]), "r"(fa[2]), "r"(fa[3]), "r"(fb[0]), "r"(fb[1]));
                }
            }
        }
        // partial tiles -> red[warp][row][token]; then one (row, token) per thread
        float *rw = red + warp * 256;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int col = nt * 8 + (int)(lane & 3u) * 2;
            const int row = (int)(lane >> 2);
            rw[row * 16 + col] = c[nt][0];
            rw[row * 16 + col + 1] = c[nt][1];
            rw[(row + 8) * 16 + col] = c[nt][2];
            rw[(row + 8) * 16 + col + 1] = c[nt][3];
        }
        __syncthreads();
        {
            const int row = threadIdx.x >> 4, t = threadIdx.x & 15;
            if (m0 + row < nrow && t < a.L) {
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < kDecodeWarps; ++w) v += red[w * 256 + threadIdx.x];
                const int g = g0 + m0 + row;
                if (g < a.N_r) a.s_r[(size_t)t * a.N_r + g] = v;
                else a.s_c[(size_t)t * a.N_c + (g - a.N_r)] = v;
            }
        }
        __syncthreads();                                    // red is rewritten next
    }
}

// The projection of two staged router rows (j0, j0 + 1 of the CTA's block,
// bf16 [rows][d] in shared memory) with the L <= LM staged token rows:
// every slice of both rows in registers, each (row, token) dot product
// reduced over the warp and written to s_r / s_c at grid row g0 + j.  LM is
// the token count rounded up to a power of two: the token loop is unrolled
// LM times, and guarded lanes of it still cost issue slots.
template <int LM>
__device__ __forceinline__ void decode_rows_dot2(const uint4 *xs, const uint4 *wsm, int j0,
                                                 int nrow, int g0, const DecodeArgs &a) {
    const int d8 = a.d >> 3;
    const unsigned lane = lane_id();
    uint4 wu[2][kSmallSlices];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int i = 0; i < kSmallSlices; ++i) {
            const int c8 = (int)lane + 32 * i;
            wu[r][i] = c8 < d8 && j0 + r < nrow ? wsm[(size_t)(j0 + r) * d8 + c8]
                                                : make_uint4(0u, 0u, 0u, 0u);
        }
    float acc[2][LM];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int t = 0; t < LM; ++t) acc[r][t] = 0.f;
#pragma unroll
    for (int i = 0; i < kSmallSlices; ++i) {
        const int c8 = (int)lane + 32 * i;
        if (c8 < d8) {
            float wf[2][8];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint32_t w4[4] = {wu[r][i].x, wu[r][i].y, wu[r][i].z, wu[r][i].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    wf[r][2 * q] = __uint_as_float(w4[q] << 16);
                    wf[r][2 * q + 1] = __uint_as_float(w4[q] & 0xffff0000u);
                }
            }
#pragma unroll
            for (int t = 0; t < LM; ++t) {
                if (t < a.L) {
                    const uint4 u = xs[(size_t)t * d8 + c8];
                    const uint32_t x4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float xlo = __uint_as_float(x4[q] << 16);
                        const float xhi = __uint_as_float(x4[q] & 0xffff0000u);
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            acc[r][t] = fmaf(xlo, wf[r][2 * q], acc[r][t]);
                            acc[r][t] = fmaf(xhi, wf[r][2 * q + 1], acc[r][t]);
                        }
                    }
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int g = g0 + j0 + r;
#pragma unroll
        for (int t = 0; t < LM; ++t) {
            if (t < a.L) {
                const float v = warp_sum(acc[r][t]);
                if (lane == 0 && j0 + r < nrow) {
                    if (g < a.N_r) a.s_r[(size_t)t * a.N_r + g] = v;
                    else a.s_c[(size_t)t * a.N_c + (g - a.N_r)] = v;
                }
            }
        }
    }
}

__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};"
                 ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

__global__ void __launch_bounds__(32 * kDecodeWarps, 2) decode_fused_kernel(const DecodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem_u[];
    __shared__ int s_ok;
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    const int d8 = a.d >> 3;

    if (blockIdx.x == 0 && threadIdx.x == 0) {
        atomicExch(a.bar, (unsigned long long)a.epoch << 32);     // this call's barrier word
        *a.status = 0;                                               // no error can precede it
    }

    // ---- A. router projection: CTA b < nproj takes rows [b rpc, (b + 1) rpc)
    // of (W_r; W_c); one bulk copy per matrix pulls them, and another the
    // token rows, into shared memory; each warp then takes two rows at a
    // time.  y zeroed unless accumulating.
    {
        const int R = a.N_r + a.N_c;
        const int r0 = (int)blockIdx.x * a.rpc;
        const int nrow = (int)blockIdx.x < a.nproj ? min(a.rpc, R - r0) : 0;
        if (nrow > 0) {
            uint4 *xs = reinterpret_cast<uint4 *>(smem_u);                      // [L][d / 8]
            uint4 *wsm = xs + (size_t)a.L * d8;                                 // [rpc][d / 8]
            uint64_t *mb = reinterpret_cast<uint64_t *>(wsm + (size_t)a.rpc * d8);
            if (threadIdx.x == 0) {
                mbar_init(mb, 1);
                fence_barrier_init();
                const uint32_t row_bytes = (uint32_t)a.d * 2u;
                const int nr = min(max(a.N_r - r0, 0), nrow);                  // rows of W_r
                mbar_arrive_expect_tx(mb, (uint32_t)a.L * row_bytes + (uint32_t)nrow * row_bytes);
                bulk_load_1d(xs, a.x, (uint32_t)a.L * row_bytes, mb);
                if (nr > 0) bulk_load_1d(wsm, a.W_r + (size_t)r0 * a.d, (uint32_t)nr * row_bytes, mb);
                if (nrow > nr)
                    bulk_load_1d(wsm + (size_t)nr * d8, a.W_c + (size_t)(r0 + nr - a.N_r) * a.d,
                                 (uint32_t)(nrow - nr) * row_bytes, mb);
            }
            __syncthreads();
            mbar_wait(mb, 0u, a.status);
            if (a.L <= 2) {
                for (int j0 = 2 * warp; j0 < nrow; j0 += 2 * kDecodeWarps) {
                    if (a.L == 1) decode_rows_dot2<1>(xs, wsm, j0, nrow, r0, a);
                    else decode_rows_dot2<2>(xs, wsm, j0, nrow, r0, a);
                }
            } else {
                decode_rows_mma(reinterpret_cast<const uint16_t *>(xs),
                                reinterpret_cast<const uint16_t *>(wsm), nrow, r0,
                                reinterpret_cast<float *>(mb + 2), a);
            }
            __syncthreads();
            if (threadIdx.x == 0)
                asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(mb)) : "memory");
        }
        if (!a.accumulate) {
            float4 *y4 = reinterpret_cast<float4 *>(a.y);
            const int n4 = a.L * (a.d >> 2);
            for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += gridDim.x * blockDim.x)
                y4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    // the candidate table of the merge, built while the projection finishes
    // elsewhere (the staged x is no longer read)
    const int t_sel = (int)gridDim.x - 1 - (int)blockIdx.x < a.L ? (int)gridDim.x - 1 - (int)blockIdx.x : -1;
    if (t_sel >= 0) {
        __syncthreads();
        merge_table(a.K, a.Kr, a.Kc, a.C, smem_u, reinterpret_cast<int *>(smem_u + a.C));
    }
    if (!decode_grid_barrier(a.bar, a.epoch, gridDim.x, a.status, &s_ok)) return;

    // ---- B. selection of token t = gridDim.x - 1 - blockIdx.x (the last
    // CTAs, which the projection reaches last): warps 0-3 the row axis and
    // warps 4-7 the column axis (named barriers 1 and 2), then the whole CTA
    // the merge; the row and column top-K pass through shared memory
    if (t_sel >= 0) {
        const int t = t_sel;
        const uint32_t *table = smem_u;
        float *lists_v = reinterpret_cast<float *>(smem_u + a.merge_head);       // [Kr + Kc]
        int *lists_i = reinterpret_cast<int *>(lists_v + a.Kr + a.Kc);          // [Kr + Kc]
        uint32_t *area = smem_u + a.merge_head + a.list_words;
        {
            const int axis = threadIdx.x >> 7;                               // 128 threads each
            const int n = axis ? a.N_c : a.N_r;
            const int kx = axis ? a.Kc : a.Kr;
            uint32_t *h = area + (size_t)axis * a.axis_words;
            uint32_t *hist = h + a.nmax_pad;
            group_axis_select((axis ? a.s_c : a.s_r) + (size_t)t * n, n, kx, threadIdx.x & 127, 128,
                              1 + axis, reinterpret_cast<float *>(h), hist, hist + kNB,
                              reinterpret_cast<uint64_t *>(hist + 2 * kNB + 8), a.tmp_cap,
                              reinterpret_cast<int *>(hist + 2 * kNB),
                              lists_v + (axis ? a.Kr : 0), lists_i + (axis ? a.Kr : 0));
        }
        __syncthreads();
        group_merge(table, lists_v, lists_i, lists_v + a.Kr, lists_i + a.Kr, a.N_c, a.K, a.Kr, a.Kc,
                    a.C, area, a.idx + (size_t)t * a.K, a.score + (size_t)t * a.K,
                    a.gate + (size_t)t * a.K);
    }
    if (!decode_grid_barrier(a.bar, a.epoch, 2 * gridDim.x, a.status, &s_ok)) return;

    // ---- C. experts: CTA b takes chunks of up to 8 tasks of one token
    // (chunk j of token t: tasks 8 j .. 8 j + 7), one per warp; each warp
    // stages its v_e row (bf16) and p = g SiLU(x_t . w_e) in shared memory,
    // then every thread sums the chunk's p v_e over its 8 columns and adds
    // them to y_t (16-byte fp32 reductions, one per 4 columns and chunk)
    uint4 *vs = reinterpret_cast<uint4 *>(smem_u);                    // [8][d / 8]
    float *ps = reinterpret_cast<float *>(vs + kDecodeWarps * d8);   // [8]
    const int kch = (a.K + kDecodeWarps - 1) / kDecodeWarps;
    for (int ch = blockIdx.x; ch < a.L * kch; ch += gridDim.x) {
        const int t = ch / kch, k0 = (ch - t * kch) * kDecodeWarps;
        const int nw = a.K - k0 < kDecodeWarps ? a.K - k0 : kDecodeWarps;
        if (warp < nw) {
            const int m = t * a.K + k0 + warp;
            int64_t e = a.idx[m];
            const float g = a.gate[m];
            if (e < 0 || e >= a.N) {
                set_status(a.status, OMNI_DEV_BAD_EXPERT);
                e = 0;
            }
            const uint4 *x4 = reinterpret_cast<const uint4 *>(a.x) + (size_t)t * d8;
            const uint4 *w4 = reinterpret_cast<const uint4 *>(a.W) + (size_t)e * d8;
            const uint4 *v4 = reinterpret_cast<const uint4 *>(a.V) + (size_t)e * d8;
            uint4 xu[kDecodeSlices], wu[kDecodeSlices], vu[kDecodeSlices];
#pragma unroll
            for (int i = 0; i < kDecodeSlices; ++i) {         // every slice in flight at once
                const int c8 = (int)lane + 32 * i;
                const bool in = c8 < d8;
                xu[i] = in ? x4[c8] : make_uint4(0u, 0u, 0u, 0u);
                wu[i] = in ? w4[c8] : make_uint4(0u, 0u, 0u, 0u);
                vu[i] = in ? v4[c8] : make_uint4(0u, 0u, 0u, 0u);
            }
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < kDecodeSlices; ++i) {
                const uint32_t xw[4] = {xu[i].x, xu[i].y, xu[i].z, xu[i].w};
                const uint32_t ww[4] = {wu[i].x, wu[i].y, wu[i].z, wu[i].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc = fmaf(__uint_as_float(xw[q] << 16), __uint_as_float(ww[q] << 16), acc);
                    acc = fmaf(__uint_as_float(xw[q] & 0xffff0000u),
                               __uint_as_float(ww[q] & 0xffff0000u), acc);
                }
            }
#pragma unroll
            for (int i = 0; i < kDecodeSlices; ++i) {
                const int c8 = (int)lane + 32 * i;
                if (c8 < d8) vs[warp * d8 + c8] = vu[i];
            }
            const float h = warp_sum(acc);
            if (lane == 0) ps[warp] = g * (h / (1.f + __expf(-h)));
        }
        __syncthreads();
        float *yr = a.y + (size_t)t * a.d;
        for (int c8 = threadIdx.x; c8 < d8; c8 += blockDim.x) {
            float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int w = 0; w < nw; ++w) {
                const uint4 u = vs[w * d8 + c8];
                const float p = ps[w];
                const uint32_t vw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    f[2 * q] = fmaf(p, __uint_as_float(vw[q] << 16), f[2 * q]);
                    f[2 * q + 1] = fmaf(p, __uint_as_float(vw[q] & 0xffff0000u), f[2 * q + 1]);
                }
            }
            red_add_v4(yr + 8 * c8, f[0], f[1], f[2], f[3]);
            red_add_v4(yr + 8 * c8 + 4, f[4], f[5], f[6], f[7]);
        }
        __syncthreads();                                   // vs and ps are rewritten next
    }
}

}  // namespace

int merge_candidates(int K, int Kr, int Kc) {
    int C = 0;
    for (int a = 0; a < Kr; ++a) {
        int nb = K / (a + 1);
        if (nb > Kc) nb = Kc;
        if (nb <= 0) break;
        C += nb;
    }
    return C;
}

template <int CAP>
static cudaError_t launch_axis_e(const float *in_r, const float *in_c, bool logsoftmax,
                                 const float *part_r, const float *part_c,
                                 float *p_r_out, float *p_c_out, int L, int N_r, int N_c, int K,
                                 float *row_val, int *row_idx, float *col_val, int *col_idx,
                                 const int *only, cudaStream_t st) {
    const int nmax = N_r > N_c ? N_r : N_c;
    const int kmax = K < nmax ? K : nmax;
    const size_t area = 2 * (size_t)kmax > 2 * (size_t)CAP ? 2 * (size_t)kmax : 2 * (size_t)CAP;
    size_t words = (((size_t)nmax + 2 * kNB + 1) & ~(size_t)1) + area;
    words = (words + 3) & ~(size_t)3;
    const size_t per_warp = words * 4;
    int wpb = (int)((64 * 1024) / per_warp);
    if (wpb > 8) wpb = 8;
    if (wpb < 1) wpb = 1;
    const size_t smem = per_warp * wpb;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(axis_topk_kernel<CAP>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t probs = 2 * (int64_t)L;
    const unsigned grid = (unsigned)((probs + wpb - 1) / wpb);
    return launch(axis_topk_kernel<CAP>, dim3(grid), dim3(32 * wpb), smem, st, in_r, in_c,
                  logsoftmax ? 1 : 0, reinterpret_cast<const float2 *>(part_r),
                  reinterpret_cast<const float2 *>(part_c), p_r_out, p_c_out, L, N_r, N_c, K,
                  row_val, row_idx, col_val, col_idx, nmax, kmax, words, only);
}

// Shared words per warp of axis_topk_reg_kernel (even): its bucket sort, or
// the exact fallback's area (axis_row_exact: the row, hist, cur and the
// selected keys and indices).
static int axis_reg_warp_words(int cap, int nmax, int kmax) {
    const int fast = 2 * kNB + 2 * cap;
    const int exact = ((nmax + 2 * kNB + 1) & ~1) + 2 * kmax;
    const int w = fast > exact ? fast : exact;
    return (w + 1) & ~1;
}

template <int NPL, int CAP>
static cudaError_t launch_axis_reg(const float *in_r, const float *in_c, int mode,
                                   const float *part_r, const float *part_c, float *p_r_out,
                                   float *p_c_out, int L, int N_r, int N_c, int K, float *row_val,
                                   int *row_idx, float *col_val, int *col_idx, cudaStream_t st) {
    constexpr int wpb = 4;
    const int nmax = N_r > N_c ? N_r : N_c;
    const int kmax = K < nmax ? K : nmax;
    const int words = axis_reg_warp_words(CAP, nmax, kmax);
    const size_t smem = (size_t)wpb * words * 4;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(axis_topk_reg_kernel<NPL, CAP>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t probs = 2 * (int64_t)L;
    const unsigned grid = (unsigned)((probs + wpb - 1) / wpb);
    return launch(axis_topk_reg_kernel<NPL, CAP>, dim3(grid), dim3(32 * wpb), smem, st, in_r, in_c,
                  mode, reinterpret_cast<const float2 *>(part_r),
                  reinterpret_cast<const float2 *>(part_c), p_r_out, p_c_out, L, N_r, N_c, K,
                  row_val, row_idx, col_val, col_idx, nmax, kmax, words);
}

template <int CAP>
static cudaError_t launch_axis_reg_npl(int npl, const float *in_r, const float *in_c, int mode,
                                       const float *part_r, const float *part_c, float *p_r_out,
                                       float *p_c_out, int L, int N_r, int N_c, int K,
                                       float *row_val, int *row_idx, float *col_val,
                                       int *col_idx, cudaStream_t st) {
#define OMNI_RG(np) return launch_axis_reg<np, CAP>(in_r, in_c, mode, part_r, part_c, p_r_out, p_c_out, L, N_r, N_c, K, row_val, row_idx, col_val, col_idx, st);
    if (npl <= 1) { OMNI_RG(1) }
    if (npl <= 2) { OMNI_RG(2) }
    if (npl <= 4) { OMNI_RG(4) }
    if (npl <= 8) { OMNI_RG(8) }
    if (npl <= 11) { OMNI_RG(11) }
    if (npl <= 12) { OMNI_RG(12) }
    OMNI_RG(16)
#undef OMNI_RG
}

cudaError_t launch_axis_topk(const float *in_r, const float *in_c, bool logsoftmax,
                             const float *part_r, const float *part_c,
                             float *p_r_out, float *p_c_out, int L, int N_r, int N_c, int K,
                             float *row_val, int *row_idx, float *col_val, int *col_idx,
                             int *flags, int *status, cudaStream_t st) {
    (void)status;
    const int nmax = N_r > N_c ? N_r : N_c;
    const int kmax = K < nmax ? K : nmax;
    const int cap = fast_capacity(kmax);
    const bool aligned = ((reinterpret_cast<uintptr_t>(in_r) | reinterpret_cast<uintptr_t>(in_c)) & 15u) == 0;
    const int npl = (nmax / 4 + 31) / 32;
    const bool reg = flags && aligned && N_r % 4 == 0 && N_c % 4 == 0 && nmax <= 2048 && cap > 0 &&
                     cap <= 320;
    const int mode = !logsoftmax ? 0 : (part_r && part_c ? 1 : 2);
    cudaError_t e;
    const int *only = nullptr;
    if (reg) {                             // the register kernel finishes every row itself
        if (cap <= 96) e = launch_axis_reg_npl<96>(npl, in_r, in_c, mode, part_r, part_c, p_r_out, p_c_out, L, N_r, N_c, K, row_val, row_idx, col_val, col_idx, st);
        else if (cap <= 192) e = launch_axis_reg_npl<192>(npl, in_r, in_c, mode, part_r, part_c, p_r_out, p_c_out, L, N_r, N_c, K, row_val, row_idx, col_val, col_idx, st);
        else e = launch_axis_reg_npl<320>(npl, in_r, in_c, mode, part_r, part_c, p_r_out, p_c_out, L, N_r, N_c, K, row_val, row_idx, col_val, col_idx, st);
        return e;
    }
#define OMNI_AX(c) return launch_axis_e<c>(in_r, in_c, logsoftmax, part_r, part_c, p_r_out, p_c_out, L, N_r, N_c, K, row_val, row_idx, col_val, col_idx, only, st);
    if (cap == 0) { OMNI_AX(0) }
    if (cap <= 96) { OMNI_AX(96) }
    if (cap <= 192) { OMNI_AX(192) }
    if (cap <= 320) { OMNI_AX(320) }
    if (cap <= 576) { OMNI_AX(576) }
    OMNI_AX(1088)
#undef OMNI_AX
}

template <int CAP>
static cudaError_t launch_merge_e(const float *row_val, const int *row_idx, const float *col_val,
                                  const int *col_idx, int L, int N_c, int K, int Kr, int Kc, int C,
                                  int32_t *idx, float *score, float *gate, const float *dead_r,
                                  const float *dead_c, int N_r, const SchedPrep *prep,
                                  cudaStream_t st) {
    SchedPrep pv;
    std::memset(&pv, 0, sizeof pv);
    if (prep) pv = *prep;
    const MergeLayout ml = merge_layout(K, Kr, Kc, C, CAP);
    const size_t head = ((size_t)C + Kr + 1 + 3) & ~(size_t)3;
    const size_t per_warp = ml.words * 4;
    // warps per CTA: the most resident warps per SM (228 KB of shared memory
    // with 1 KB reserved per CTA, 48 registers per thread, 64 warps), fewest
    // warps per CTA on a tie
    int wpb = 1, best = 0;
    for (int w = 1; w <= 8; ++w) {
        const size_t smem = head * 4 + per_warp * (size_t)w;
        if (smem > 227 * 1024) break;
        int ctas = (int)((228 * 1024) / (smem + 1024));
        const int by_regs = 65536 / (48 * 32 * w);
        if (ctas > by_regs) ctas = by_regs;
        if (ctas > 32) ctas = 32;
        int warps = ctas * w;
        if (warps > 64) warps = 64;
        if (warps > best) {
            best = warps;
            wpb = w;
        }
    }
    const size_t smem = head * 4 + per_warp * wpb;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(merge_topk_kernel<CAP>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    const unsigned grid = (unsigned)((L + wpb - 1) / wpb);
    return launch(merge_topk_kernel<CAP>, dim3(grid), dim3(32 * wpb), smem, st, row_val, row_idx,
                  col_val, col_idx, L, N_c, K, Kr, Kc, C, idx, score, gate, dead_r, dead_c, N_r,
                  pv);
}

cudaError_t launch_merge_topk(const float *row_val, const int *row_idx, const float *col_val,
                              const int *col_idx, int L, int N_c, int K, int Kr, int Kc, int C,
                              int32_t *idx, float *score, float *gate, const float *dead_r,
                              const float *dead_c, int N_r, const SchedPrep *prep,
                              cudaStream_t st) {
    int cap = fast_capacity(K);
    if (cap > C) cap = C >= K ? (C / 32) * 32 : 0;
#define OMNI_MG(c) return launch_merge_e<c>(row_val, row_idx, col_val, col_idx, L, N_c, K, Kr, Kc, C, idx, score, gate, dead_r, dead_c, N_r, prep, st);
    if (cap < K) { OMNI_MG(0) }
    if (cap <= 96) { OMNI_MG(96) }
    if (cap <= 128) { OMNI_MG(128) }
    if (cap <= 192) { OMNI_MG(192) }
    if (cap <= 320) { OMNI_MG(320) }
    if (cap <= 576) { OMNI_MG(576) }
    OMNI_MG(1088)
#undef OMNI_MG
}

// Candidates the axis bucket sort of the fused decode step takes (more go to
// its radix select).
static int decode_tmp_cap(int nmax, int kmax) {
    const int cap = nmax < 1024 ? nmax : 1024;
    return cap > kmax ? cap : kmax;
}

// Shared words of one axis half of the fused decode step (group_axis_select):
// the row (nmax, rounded up to even), hist and cur (kNB each), 8 words of
// scratch and the 64-bit candidate keys; a multiple of 4.
static size_t decode_axis_words(int nmax, int kmax) {
    const size_t words = (((size_t)nmax + 1) & ~(size_t)1) + 2 * kNB + 8 +
                         2 * (size_t)decode_tmp_cap(nmax, kmax);
    return (words + 3) & ~(size_t)3;
}

// Shared words of the block-wide merge (group_merge): its head and the
// 64-bit keys of the C candidates.
static size_t decode_merge_words(int K, int C) {
    return ((size_t)group_merge_head_words(K) + 2 * (size_t)C + 3) & ~(size_t)3;
}

// Shared words of a token's row and column top-K lists (values and indices),
// a multiple of 4.
static size_t decode_list_words(int Kr, int Kc) {
    return ((size_t)2 * (Kr + Kc) + 3) & ~(size_t)3;
}

// The launch shape of the fused decode step for these sizes: two CTAs per SM
// when their shared memory allows it, else one; the first grid - L CTAs
// project rpc router rows each (the last L select, one token each).  Shared
// memory per CTA is the largest of phase A (token rows, router rows, the
// copy barrier), phase B (candidate table, the token's lists, the axis
// halves or the merge) and phase C (8 staged v rows and their p).
struct DecodePlan {
    int grid, rpc, nproj;
    size_t smem;
};

static bool decode_plan(int L, int d, int N_r, int N_c, int K, int Kr, int Kc, int C,
                        DecodePlan *plan) {
    if (L < 1 || L > 16 || K > 128 || d > 32 * 8 * kSmallSlices || d % 256 != 0) return false;
    const int nmax = N_r > N_c ? N_r : N_c;
    const int kmax = Kr > Kc ? Kr : Kc;
    const size_t axis_words = decode_axis_words(nmax, kmax);
    const size_t head = ((size_t)C + Kr + 1 + 3) & ~(size_t)3;
    const size_t mw = decode_merge_words(K, C);
    const size_t area = 2 * axis_words > mw ? 2 * axis_words : mw;
    const size_t lists = decode_list_words(Kr, Kc);
    const size_t b_bytes = 4 * (head + lists + area);
    const size_t c_bytes = (size_t)kDecodeWarps * d * 2 + 4 * kDecodeWarps;
    const int sms = device_sm_count();
    for (int per_sm = 2; per_sm >= 1; --per_sm) {
        const int grid = sms * per_sm;
        const int nproj = grid - L;
        if (nproj < 1) continue;
        const int rpc = (N_r + N_c + nproj - 1) / nproj;
        const size_t a_bytes = (size_t)(L + rpc) * d * 2 + 16 + 4 * 256 * kDecodeWarps;
        size_t bytes = a_bytes > b_bytes ? a_bytes : b_bytes;
        if (c_bytes > bytes) bytes = c_bytes;
        if (bytes > 200 * 1024) continue;
        if (per_sm == 2 && 2 * (bytes + 1024) > 228 * 1024) continue;
        *plan = {grid, rpc, nproj, bytes};
        return true;
    }
    return false;
}

// The plan for these sizes, with every CTA of its grid resident at once on
// this device (a cooperative launch needs that); false otherwise, and the
// routed forward then takes the separate kernels.
static bool decode_plan_resident(int L, int d, int N_r, int N_c, int K, int Kr, int Kc, int C,
                                 DecodePlan *plan) {
    if (!decode_plan(L, d, N_r, N_c, K, Kr, Kc, C, plan)) return false;
    if (cudaFuncSetAttribute(decode_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)plan->smem) != cudaSuccess)
        return false;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_fused_kernel,
                                                      32 * kDecodeWarps, plan->smem) != cudaSuccess)
        return false;
    return per_sm * device_sm_count() >= plan->grid;
}

bool decode_fused_ok(int L, int d, int N_r, int N_c, int K, int Kr, int Kc, int C) {
    DecodePlan plan;
    return decode_plan_resident(L, d, N_r, N_c, K, Kr, Kc, C, &plan);
}

cudaError_t launch_decode_fused(const uint16_t *x, const uint16_t *W, const uint16_t *V,
                                const uint16_t *W_r, const uint16_t *W_c, int L, int d, int N_r,
                                int N_c, int K, int Kr, int Kc, int C, float *s_r, float *s_c,
                                float *row_val, int *row_idx, float *col_val, int *col_idx,
                                int32_t *idx, float *score, float *gate, float *y,
                                bool accumulate, unsigned long long *bar, unsigned epoch,
                                int *status, cudaStream_t st) {
    DecodePlan plan;
    if (!decode_plan_resident(L, d, N_r, N_c, K, Kr, Kc, C, &plan)) return cudaErrorInvalidValue;
    DecodeArgs a;
    a.x = x; a.W = W; a.V = V; a.W_r = W_r; a.W_c = W_c;
    a.L = L; a.d = d; a.N_r = N_r; a.N_c = N_c; a.K = K; a.Kr = Kr; a.Kc = Kc; a.C = C;
    a.N = (int64_t)N_r * N_c;
    a.s_r = s_r; a.s_c = s_c; a.row_val = row_val; a.col_val = col_val;
    a.row_idx = row_idx; a.col_idx = col_idx; a.idx = idx; a.score = score; a.gate = gate;
    a.y = y; a.accumulate = accumulate ? 1 : 0; a.bar = bar; a.epoch = epoch; a.status = status;
    a.rpc = plan.rpc; a.nproj = plan.nproj;
    a.nmax = N_r > N_c ? N_r : N_c;
    a.kmax = Kr > Kc ? Kr : Kc;
    a.axis_words = (int)decode_axis_words(a.nmax, a.kmax);
    a.merge_head = (int)(((size_t)C + Kr + 1 + 3) & ~(size_t)3);
    a.list_words = (int)decode_list_words(Kr, Kc);
    a.nmax_pad = (a.nmax + 1) & ~1;
    a.tmp_cap = decode_tmp_cap(a.nmax, a.kmax);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)plan.grid);
    cfg.blockDim = dim3(32 * kDecodeWarps);
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    first_launch_in_call();                     // ordinary stream order for what follows it too
    return cudaLaunchKernelEx(&cfg, decode_fused_kernel, a);
}

}  // namespace omni

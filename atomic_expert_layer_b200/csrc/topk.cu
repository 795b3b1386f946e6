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
        float mx = -INFINITY;
        for (int i = lane; i < n; i += 32) {
            const float v = in[i];
            vals[i] = v;
            mx = fmaxf(mx, v);
        }
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
// computed here.  A row this kernel cannot finish (too few values within 8
// units of the maximum, or more than CAP candidates) sets flags[row] = 1 and
// is redone by axis_topk_kernel; every other row gets flags[row] = 0.
// Shared memory per warp (words): hist[kNB] | cur[kNB] | tmp[CAP] (u64).
template <int NPL, int CAP>
__global__ void __launch_bounds__(128)
axis_topk_reg_kernel(const float *__restrict__ in_r, const float *__restrict__ in_c, int mode,
                     const float2 *__restrict__ part_r, const float2 *__restrict__ part_c,
                     float *__restrict__ p_r_out, float *__restrict__ p_c_out, int L, int N_r,
                     int N_c, int K, float *__restrict__ row_val, int *__restrict__ row_idx,
                     float *__restrict__ col_val, int *__restrict__ col_idx,
                     int *__restrict__ flags) {
    extern __shared__ __align__(16) uint32_t smem_u[];
    constexpr int kWords = 2 * kNB + 2 * CAP;
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
    uint32_t *hist = smem_u + (size_t)warp * kWords;
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
    if (ncand < kx || ncand > CAP) {
        if (lane == 0) flags[prob] = 1;
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
    float *oval = (axis ? col_val : row_val) + (size_t)t * kx;
    int *oidx = (axis ? col_idx : row_idx) + (size_t)t * kx;
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
    if (lane == 0) flags[prob] = 0;
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

// ------------------------------------------------------- fused decode step
// For a handful of tokens the routed forward is latency-bound: six dependent
// launches, each starting cold, cost about 37 us at L = 1 against a 1.7 us
// roofline.  Tokens are independent once the router projection is done, so
// one cooperative launch (every CTA resident) runs the whole step in three
// phases separated by a grid barrier (a bounded wait):
//   A. all CTAs: the streamed router projection (small_rows_dot, the
//      arithmetic of the small-batch projection kernel) into s; y zeroed
//      unless accumulating;
//   B. CTA t < L, token t: LogSoftmax and the exact row and column top-K
//      (warps 0 and 1, axis_row_exact), then the merge and the gates (warp 0,
//      merge_token): the same selection as the separate kernels;
//   C. every warp, one task (t, k) at a time in token order: h = x_t . w_e,
//      p = g SiLU(h), y_t += p v_e (16-byte fp32 reductions; the order in
//      which a token's K terms land varies from run to run).
constexpr int kDecodeWarps = 8;
constexpr int kDecodeCap = 192;            // axis and merge fast-path capacity (K <= 128)
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
    unsigned *bar;                         // zeroed per call
    int *status;
    int nmax, kmax;
    int axis_words;                        // shared words per axis warp
    int merge_head;                        // candidate table and its scratch
};

// All CTAs of the grid arrive; the wait gives up after kWaitLimitNs and
// records OMNI_DEV_WAIT_TIMEOUT (then the CTA returns).
__device__ bool decode_grid_barrier(unsigned *bar, unsigned target, int *status, int *s_ok) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(bar, 1u);
        bool ok = true;
        const uint64_t t0 = global_timer_ns();
        for (uint32_t it = 0;; ++it) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
            if (v >= target) break;
            if ((it & 63u) == 63u &&
                (it > kWaitSpinLimit || global_timer_ns() - t0 > kWaitLimitNs)) {
                set_status(status, OMNI_DEV_WAIT_TIMEOUT);
                ok = false;
                break;
            }
        }
        *s_ok = ok ? 1 : 0;
    }
    __syncthreads();
    return *s_ok != 0;
}

__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};"
                 ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

__global__ void __launch_bounds__(32 * kDecodeWarps) decode_fused_kernel(const DecodeArgs a) {
    extern __shared__ __align__(16) uint32_t smem_u[];
    __shared__ int s_ok;
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    const int d8 = a.d >> 3;

    // ---- A. router projection; y zeroed
    {
        uint4 *xs = reinterpret_cast<uint4 *>(smem_u);            // [L][d / 8]
        const int nblk = (a.N_r + a.N_c + kSmallRows - 1) / kSmallRows;
        bool staged = false;
        for (int blk0 = blockIdx.x * kDecodeWarps; blk0 < nblk;
             blk0 += gridDim.x * kDecodeWarps) {                    // the same in every warp
            small_rows_dot<16>(xs, a.W_r, a.W_c, a.L, a.d, a.N_r, a.N_c,
                               (blk0 + warp) * kSmallRows, a.s_r, a.s_c, [&]() {
                if (!staged) {
                    for (int i = threadIdx.x; i < a.L * d8; i += blockDim.x)
                        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                                     ::"r"(smem_u32(xs + i)),
                                     "l"(reinterpret_cast<const uint4 *>(a.x) + i)
                                     : "memory");
                    asm volatile("cp.async.commit_group;" ::: "memory");
                    asm volatile("cp.async.wait_group 0;" ::: "memory");
                    __syncthreads();
                    staged = true;
                }
            });
        }
        if (!a.accumulate) {
            float4 *y4 = reinterpret_cast<float4 *>(a.y);
            const int n4 = a.L * (a.d >> 2);
            for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += gridDim.x * blockDim.x)
                y4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    if (!decode_grid_barrier(a.bar, gridDim.x, a.status, &s_ok)) return;

    // ---- B. selection of token t = blockIdx.x
    if ((int)blockIdx.x < a.L) {
        const int t = blockIdx.x;
        uint32_t *table = smem_u;
        merge_table(a.K, a.Kr, a.Kc, a.C, table, reinterpret_cast<int *>(table + a.C));
        uint32_t *area = smem_u + a.merge_head;
        if (warp < 2) {
            const int axis = warp;
            const int n = axis ? a.N_c : a.N_r;
            const int kx = axis ? a.Kc : a.Kr;
            axis_row_exact<kDecodeCap>((axis ? a.s_c : a.s_r) + (size_t)t * n, n, kx, 1, nullptr, t,
                                       nullptr, (axis ? a.col_val : a.row_val) + (size_t)t * kx,
                                       (axis ? a.col_idx : a.row_idx) + (size_t)t * kx, a.nmax,
                                       a.kmax, area + (size_t)axis * a.axis_words);
        }
        __syncthreads();
        if (warp == 0) {
            const MergeLayout ml = merge_layout(a.K, a.Kr, a.Kc, a.C, kDecodeCap);
            const SchedPrep none{};
            merge_token<kDecodeCap>(table, area, ml, a.row_val + (size_t)t * a.Kr,
                                    a.row_idx + (size_t)t * a.Kr, a.col_val + (size_t)t * a.Kc,
                                    a.col_idx + (size_t)t * a.Kc, a.N_c, a.K, a.Kr, a.Kc, a.C, t,
                                    a.idx + (size_t)t * a.K, a.score + (size_t)t * a.K,
                                    a.gate + (size_t)t * a.K, none);
        }
    }
    if (!decode_grid_barrier(a.bar, 2 * gridDim.x, a.status, &s_ok)) return;

    // ---- C. experts, one task per warp at a time
    const int nwarps = gridDim.x * kDecodeWarps;
    for (int m = blockIdx.x * kDecodeWarps + warp; m < a.L * a.K; m += nwarps) {
        const int t = m / a.K;
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
        for (int i = 0; i < kDecodeSlices; ++i) {             // every slice in flight at once
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
                acc = fmaf(__uint_as_float(xw[q] & 0xffff0000u), __uint_as_float(ww[q] & 0xffff0000u),
                           acc);
            }
        }
        const float h = warp_sum(acc);
        const float p = g * (h / (1.f + __expf(-h)));
        float *yr = a.y + (size_t)t * a.d;
#pragma unroll
        for (int i = 0; i < kDecodeSlices; ++i) {
            const int c8 = (int)lane + 32 * i;
            if (c8 < d8) {
                const uint32_t vw[4] = {vu[i].x, vu[i].y, vu[i].z, vu[i].w};
                float f[8];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    f[2 * q] = p * __uint_as_float(vw[q] << 16);
                    f[2 * q + 1] = p * __uint_as_float(vw[q] & 0xffff0000u);
                }
                red_add_v4(yr + 8 * c8, f[0], f[1], f[2], f[3]);
                red_add_v4(yr + 8 * c8 + 4, f[4], f[5], f[6], f[7]);
            }
        }
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

template <int NPL, int CAP>
static cudaError_t launch_axis_reg(const float *in_r, const float *in_c, int mode,
                                   const float *part_r, const float *part_c, float *p_r_out,
                                   float *p_c_out, int L, int N_r, int N_c, int K, float *row_val,
                                   int *row_idx, float *col_val, int *col_idx, int *flags,
                                   cudaStream_t st) {
    constexpr int wpb = 4;
    const size_t smem = (size_t)wpb * (2 * kNB + 2 * CAP) * 4;
    const int64_t probs = 2 * (int64_t)L;
    const unsigned grid = (unsigned)((probs + wpb - 1) / wpb);
    return launch(axis_topk_reg_kernel<NPL, CAP>, dim3(grid), dim3(32 * wpb), smem, st, in_r, in_c,
                  mode, reinterpret_cast<const float2 *>(part_r),
                  reinterpret_cast<const float2 *>(part_c), p_r_out, p_c_out, L, N_r, N_c, K,
                  row_val, row_idx, col_val, col_idx, flags);
}

template <int CAP>
static cudaError_t launch_axis_reg_npl(int npl, const float *in_r, const float *in_c, int mode,
                                       const float *part_r, const float *part_c, float *p_r_out,
                                       float *p_c_out, int L, int N_r, int N_c, int K,
                                       float *row_val, int *row_idx, float *col_val,
                                       int *col_idx, int *flags, cudaStream_t st) {
#define OMNI_RG(np) return launch_axis_reg<np, CAP>(in_r, in_c, mode, part_r, part_c, p_r_out, p_c_out, L, N_r, N_c, K, row_val, row_idx, col_val, col_idx, flags, st);
    if (npl <= 1) { OMNI_RG(1) }
    if (npl <= 2) { OMNI_RG(2) }
    if (npl <= 4) { OMNI_RG(4) }
    if (npl <= 8) { OMNI_RG(8) }
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
    if (reg) {
        if (cap <= 96) e = launch_axis_reg_npl<96>(npl, in_r, in_c, mode, part_r, part_c, p_r_out, p_c_out, L, N_r, N_c, K, row_val, row_idx, col_val, col_idx, flags, st);
        else if (cap <= 192) e = launch_axis_reg_npl<192>(npl, in_r, in_c, mode, part_r, part_c, p_r_out, p_c_out, L, N_r, N_c, K, row_val, row_idx, col_val, col_idx, flags, st);
        else e = launch_axis_reg_npl<320>(npl, in_r, in_c, mode, part_r, part_c, p_r_out, p_c_out, L, N_r, N_c, K, row_val, row_idx, col_val, col_idx, flags, st);
        if (e != cudaSuccess) return e;
        only = flags;                      // the general kernel redoes the flagged rows
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

// Shared words of one axis warp of the fused decode step: axis_row_exact's
// values, two bucket arrays and max(2 kmax, 2 CAP) words of candidates (as
// the stand-alone axis kernel takes), a multiple of 4.
static size_t decode_axis_words(int nmax, int kmax) {
    const size_t area = kmax > kDecodeCap ? 2 * (size_t)kmax : 2 * (size_t)kDecodeCap;
    const size_t words = (((size_t)nmax + 2 * kNB + 1) & ~(size_t)1) + area;
    return (words + 3) & ~(size_t)3;
}

// Shared words of the fused decode step for these sizes (0 if it does not
// apply): the larger of phase A (x) and phase B (candidate table, two axis
// warps or the merge warp).
static size_t decode_smem_bytes(int L, int d, int N_r, int N_c, int K, int Kr, int Kc, int C) {
    if (L > 16 || K > 128 || d > 32 * 8 * kDecodeSlices || d % 256 != 0) return 0;
    const int nmax = N_r > N_c ? N_r : N_c;
    const int kmax = Kr > Kc ? Kr : Kc;
    const size_t axis_words = decode_axis_words(nmax, kmax);
    const size_t head = ((size_t)C + Kr + 1 + 3) & ~(size_t)3;
    const MergeLayout ml = merge_layout(K, Kr, Kc, C, kDecodeCap);
    const size_t area = 2 * axis_words > ml.words ? 2 * axis_words : ml.words;
    const size_t b_bytes = 4 * (head + area);
    const size_t a_bytes = (size_t)L * d * 2;
    const size_t bytes = a_bytes > b_bytes ? a_bytes : b_bytes;
    return bytes <= 200 * 1024 ? bytes : 0;
}

bool decode_fused_ok(int L, int d, int N_r, int N_c, int K, int Kr, int Kc, int C) {
    return decode_smem_bytes(L, d, N_r, N_c, K, Kr, Kc, C) > 0;
}

cudaError_t launch_decode_fused(const uint16_t *x, const uint16_t *W, const uint16_t *V,
                                const uint16_t *W_r, const uint16_t *W_c, int L, int d, int N_r,
                                int N_c, int K, int Kr, int Kc, int C, float *s_r, float *s_c,
                                float *row_val, int *row_idx, float *col_val, int *col_idx,
                                int32_t *idx, float *score, float *gate, float *y,
                                bool accumulate, unsigned *bar, int *status, cudaStream_t st) {
    const size_t smem = decode_smem_bytes(L, d, N_r, N_c, K, Kr, Kc, C);
    if (smem == 0) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(decode_fused_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_fused_kernel,
                                                      32 * kDecodeWarps, smem);
    if (e != cudaSuccess) return e;
    if (per_sm > 2) per_sm = 2;
    const int grid = device_sm_count() * per_sm;      // every CTA resident (cooperative launch)
    if (per_sm < 1 || grid < L) return cudaErrorInvalidValue;
    DecodeArgs a;
    a.x = x; a.W = W; a.V = V; a.W_r = W_r; a.W_c = W_c;
    a.L = L; a.d = d; a.N_r = N_r; a.N_c = N_c; a.K = K; a.Kr = Kr; a.Kc = Kc; a.C = C;
    a.N = (int64_t)N_r * N_c;
    a.s_r = s_r; a.s_c = s_c; a.row_val = row_val; a.col_val = col_val;
    a.row_idx = row_idx; a.col_idx = col_idx; a.idx = idx; a.score = score; a.gate = gate;
    a.y = y; a.accumulate = accumulate ? 1 : 0; a.bar = bar; a.status = status;
    a.nmax = N_r > N_c ? N_r : N_c;
    a.kmax = Kr > Kc ? Kr : Kc;
    a.axis_words = (int)decode_axis_words(a.nmax, a.kmax);
    a.merge_head = (int)(((size_t)C + Kr + 1 + 3) & ~(size_t)3);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(32 * kDecodeWarps);
    cfg.dynamicSmemBytes = smem;
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

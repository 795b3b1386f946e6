// backward.cu -- backward of the routed branch on sm_100a.
//
// "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale" gives
// the forward only (rainbus review page, method paragraph, steps 1-3); this is
// its derivative with the top-K selection held fixed.  For token t and task k
// (expert e = idx[t,k] at grid cell (i, j) = (e / N_c, e % N_c), gate g):
//   h = x_t . w_e,  a = SiLU(h),  c = dy_t . v_e
//   dgate_k = a c,   dV[e] += g a dy_t,
//   dh = g c SiLU'(h),   dW[e] += dh x_t,   dx_t += dh w_e
// gates are a softmax over the token's K scores S, so
//   dS_k = g_k (dgate_k - sum_j g_j dgate_j),
// S = p_r[i] + p_c[j] sends dS_k to dp_r[i] and dp_c[j], and the LogSoftmax
// p = s - logsumexp(s) gives ds = dp - softmax(s) * sum(dp).  sum(dp) is
// sum_k dS_k = sum g dgate - (sum g)(sum g dgate) = 0 because the selected
// gates sum to 1, so ds = dp exactly and the router gradient is sparse:
//   dx_t += sum_i dp_r[i] W_r[i] + sum_j dp_c[j] W_c[j],
//   dW_r[i] += dp_r[i] x_t,  dW_c[j] += dp_c[j] x_t.
//
// One warp per token: x_t and dy_t stay in registers, the K expert rows of W
// and V are gathered, dx_t is accumulated in registers and written once.  The
// dW and dV rows of an expert that only this task uses (most of them, when
// the tasks spread over many experts) get a plain read-add-write; the others
// are scatter-added with 16-byte fp32 reductions, which the L2 runs well
// below HBM bandwidth.  A first kernel marks the experts used more than once
// (two bitmaps over the N experts) when the workspace has room for them.
// The router rows are touched once per distinct row / column of the token (its
// K cells sit in few rows and columns, (a+1)(b+1) <= K).  With room in the
// workspace, the token stores (t, dS) in that row's slot list instead of
// reducing dS x_t onto it; a second kernel then sums each list and adds it to
// its dW_r / dW_c row once.  A pair that finds its list full, or every pair
// when there are no lists, is reduced into the row in fp32.
#include "omni_common.cuh"
#include "omni_internal.h"

namespace omni {
namespace {

constexpr int kBwdWarps = 4;
constexpr int kPrefetch = 1;              // tasks whose rows are asked of L2 ahead (2 measured slower)

__device__ __forceinline__ void bf16x8_f32(const uint4 &u, float *f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ void red_add_f32x4(float *gaddr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};"
                 ::"l"(gaddr), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

// row += s * (this lane's 8 * VPL columns, column (v * 32 + lane) * 8 + c),
// the values given as fp32 (f) or as raw bf16 (u)
template <int VPL>
__device__ __forceinline__ void red_row_f32(float *row, float s, const float *f, unsigned lane) {
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        float *p = row + (size_t)(v * 32 + lane) * 8;
        const float *q = f + 8 * v;
        red_add_f32x4(p, s * q[0], s * q[1], s * q[2], s * q[3]);
        red_add_f32x4(p + 4, s * q[4], s * q[5], s * q[6], s * q[7]);
    }
}
template <int VPL>
__device__ __forceinline__ void red_row_bf16(float *row, float s, const uint4 *u, unsigned lane) {
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        float q[8];
        bf16x8_f32(u[v], q);
        float *p = row + (size_t)(v * 32 + lane) * 8;
        red_add_f32x4(p, s * q[0], s * q[1], s * q[2], s * q[3]);
        red_add_f32x4(p + 4, s * q[4], s * q[5], s * q[6], s * q[7]);
    }
}
// The same two updates as a plain read-add-write, for a row no other task
// touches (both rows are read before either is written back).
template <int VPL>
__device__ __forceinline__ void rmw_rows(float *rv, float sv, const float *fv, float *rw, float sw,
                                         const uint4 *uw, unsigned lane) {
    float4 ov[2 * VPL], ow[2 * VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        const float4 *pv = reinterpret_cast<const float4 *>(rv + (size_t)(v * 32 + lane) * 8);
        const float4 *pw = reinterpret_cast<const float4 *>(rw + (size_t)(v * 32 + lane) * 8);
        ov[2 * v] = pv[0];
        ov[2 * v + 1] = pv[1];
        ow[2 * v] = pw[0];
        ow[2 * v + 1] = pw[1];
    }
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        const float *q = fv + 8 * v;
        float w[8];
        bf16x8_f32(uw[v], w);
        float4 *pv = reinterpret_cast<float4 *>(rv + (size_t)(v * 32 + lane) * 8);
        float4 *pw = reinterpret_cast<float4 *>(rw + (size_t)(v * 32 + lane) * 8);
        pv[0] = make_float4(fmaf(sv, q[0], ov[2 * v].x), fmaf(sv, q[1], ov[2 * v].y),
                            fmaf(sv, q[2], ov[2 * v].z), fmaf(sv, q[3], ov[2 * v].w));
        pv[1] = make_float4(fmaf(sv, q[4], ov[2 * v + 1].x), fmaf(sv, q[5], ov[2 * v + 1].y),
                            fmaf(sv, q[6], ov[2 * v + 1].z), fmaf(sv, q[7], ov[2 * v + 1].w));
        pw[0] = make_float4(fmaf(sw, w[0], ow[2 * v].x), fmaf(sw, w[1], ow[2 * v].y),
                            fmaf(sw, w[2], ow[2 * v].z), fmaf(sw, w[3], ow[2 * v].w));
        pw[1] = make_float4(fmaf(sw, w[4], ow[2 * v + 1].x), fmaf(sw, w[5], ow[2 * v + 1].y),
                            fmaf(sw, w[6], ow[2 * v + 1].z), fmaf(sw, w[7], ow[2 * v + 1].w));
    }
}

// acc += s * (raw bf16 slice u)
template <int VPL>
__device__ __forceinline__ void axpy_bf16(float *acc, float s, const uint4 *u) {
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        float q[8];
        bf16x8_f32(u[v], q);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[8 * v + c] = fmaf(s, q[c], acc[8 * v + c]);
    }
}
// Asks L2 for the 128-byte lines of a row of `bytes` bytes (one line per
// lane and round), so that a later load of it does not wait for HBM.
__device__ __forceinline__ void prefetch_row_l2(const void *row, int bytes, unsigned lane) {
    const char *p = static_cast<const char *>(row);
    for (int o = (int)lane * 128; o < bytes; o += 32 * 128)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(p + o));
}

template <int VPL>
__device__ __forceinline__ void load_raw(const uint16_t *row, uint4 *u, unsigned lane) {
    const uint4 *r4 = reinterpret_cast<const uint4 *>(row);
#pragma unroll
    for (int v = 0; v < VPL; ++v) u[v] = r4[v * 32 + lane];
}

// Sorts the K pairs (key[k], val[k]) by key (ties by k), adds val over equal
// keys, and writes the n distinct keys to key[0, n) and their sums to
// out[0, n) in key order; returns n.  ord and tmp are K-entry scratch; val
// is only read.  One warp; the sums run in a fixed order.
__device__ int combine_by_key(int *key, const float *val, int *ord, float *tmp, float *out,
                              int K) {
    const unsigned lane = lane_id();
    for (int k = lane; k < K; k += 32) {
        const int r = key[k];
        int rank = 0;
        for (int m = 0; m < K; ++m) {
            const int rm = key[m];
            rank += (rm < r) | ((rm == r) & (m < k));
        }
        ord[rank] = k;                                  // ranks form a permutation
    }
    __syncwarp();
    for (int p = lane; p < K; p += 32) {               // each lane its own positions
        const int k = ord[p];
        tmp[p] = val[k];
        ord[p] = key[k];                                // ord now holds sorted keys
    }
    __syncwarp();
    int n = 0;
    for (int p0 = 0; p0 < K; p0 += 32) {
        const int p = p0 + (int)lane;
        const bool head = p < K && (p == 0 || ord[p] != ord[p - 1]);
        float s = 0.f;
        int r = 0;
        if (head) {
            r = ord[p];
            for (int q = p; q < K && ord[q] == r; ++q) s += tmp[q];
        }
        const unsigned bal = __ballot_sync(0xffffffffu, head);
        if (head) {                                     // pos <= p: no read is overwritten
            const int pos = n + __popc(bal & lanemask_lt());
            key[pos] = r;
            out[pos] = s;
        }
        n += __popc(bal);
    }
    __syncwarp();
    return n;
}

template <int VPL>
__global__ void __launch_bounds__(32 * kBwdWarps)
routed_bwd_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ W,
                  const uint16_t *__restrict__ V, const uint16_t *__restrict__ W_r,
                  const uint16_t *__restrict__ W_c, int L, int N, int N_c, int K,
                  const int32_t *__restrict__ idx, const float *__restrict__ gate,
                  const float *__restrict__ dy, float *__restrict__ dx, float *__restrict__ dW,
                  float *__restrict__ dV, float *__restrict__ dW_r, float *__restrict__ dW_c,
                  const uint32_t *__restrict__ shared_rows, int *__restrict__ rcnt,
                  int2 *__restrict__ rslots, int rcap, int N_r, int *status) {
    constexpr int D = 256 * VPL;
    constexpr int E = 8 * VPL;                       // columns per lane
    extern __shared__ __align__(16) uint8_t smem[];
    grid_dependency_wait();
    grid_dependents_launch();
    const int warp = threadIdx.x >> 5;
    const unsigned lane = lane_id();
    // per warp, K entries each: expert, gate (later: combined sums), dS, key, order, scratch
    int *se = reinterpret_cast<int *>(smem) + (size_t)warp * 6 * K;
    float *sg = reinterpret_cast<float *>(se + K);
    float *sd = sg + K;
    int *key = reinterpret_cast<int *>(sd + K);
    int *ord = key + K;
    float *tmp = reinterpret_cast<float *>(ord + K);
    const int t = blockIdx.x * kBwdWarps + warp;
    if (t >= L) return;                              // the same in every lane

    for (int k = lane; k < K; k += 32) {
        int e = idx[(size_t)t * K + k];
        if (e < 0 || e >= N) {
            set_status(status, OMNI_DEV_BAD_EXPERT);
            e = 0;
        }
        se[k] = e;
        sg[k] = gate[(size_t)t * K + k];
    }
    __syncwarp();
    uint4 xu[VPL];
    load_raw<VPL>(x + (size_t)t * D, xu, lane);
    float dyf[E], acc[E];
    {
        const float4 *d4 = reinterpret_cast<const float4 *>(dy + (size_t)t * D);
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            const float4 a = d4[(v * 32 + lane) * 2], b = d4[(v * 32 + lane) * 2 + 1];
            dyf[8 * v] = a.x; dyf[8 * v + 1] = a.y; dyf[8 * v + 2] = a.z; dyf[8 * v + 3] = a.w;
            dyf[8 * v + 4] = b.x; dyf[8 * v + 5] = b.y; dyf[8 * v + 6] = b.z; dyf[8 * v + 7] = b.w;
        }
    }
#pragma unroll
    for (int c = 0; c < E; ++c) acc[c] = 0.f;

    // ---- expert part
    float sgd = 0.f;                                 // sum_k g_k dgate_k (same in every lane)
    for (int k = 0; k < K; ++k) {
        const int e = se[k];
        const float g = sg[k];
        // the rows of the task kPrefetch ahead, into L2 (the first ones
        // before the loop)
        for (int kk = k == 0 ? 1 : k + kPrefetch; kk <= k + kPrefetch && kk < K; ++kk) {
            const int en = se[kk];
            prefetch_row_l2(W + (size_t)en * D, 2 * D, lane);
            prefetch_row_l2(V + (size_t)en * D, 2 * D, lane);
            prefetch_row_l2(dW + (size_t)en * D, 4 * D, lane);
            prefetch_row_l2(dV + (size_t)en * D, 4 * D, lane);
        }
        // an expert no other task uses gets a plain read-add-write of its rows
        const bool own = shared_rows && !((shared_rows[e >> 5] >> (e & 31)) & 1u);
        uint4 wu[VPL], vu[VPL];
        load_raw<VPL>(W + (size_t)e * D, wu, lane);
        load_raw<VPL>(V + (size_t)e * D, vu, lane);
        float h = 0.f, c = 0.f;
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            float xq[8], wq[8], vq[8];
            bf16x8_f32(xu[v], xq);
            bf16x8_f32(wu[v], wq);
            bf16x8_f32(vu[v], vq);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                h = fmaf(xq[q], wq[q], h);
                c = fmaf(dyf[8 * v + q], vq[q], c);
            }
        }
        h = warp_sum(h);
        c = warp_sum(c);
        const float s = 1.f / (1.f + __expf(-h));
        const float a = h * s;
        const float dg = a * c;
        const float dh = g * c * (s * (1.f + h * (1.f - s)));
        if (own) {
            rmw_rows<VPL>(dV + (size_t)e * D, g * a, dyf, dW + (size_t)e * D, dh, xu, lane);
        } else {
            red_row_f32<VPL>(dV + (size_t)e * D, g * a, dyf, lane);
            red_row_bf16<VPL>(dW + (size_t)e * D, dh, xu, lane);
        }
        axpy_bf16<VPL>(acc, dh, wu);
        if (lane == 0) sd[k] = dg;
        sgd = fmaf(g, dg, sgd);
    }
    __syncwarp();
    // dS_k = g_k (dgate_k - sum_j g_j dgate_j)
    for (int k = lane; k < K; k += 32) sd[k] = sg[k] * (sd[k] - sgd);
    __syncwarp();

    // ---- router part: rows, then columns, each distinct one once
    for (int axis = 0; axis < 2; ++axis) {
        for (int k = lane; k < K; k += 32) key[k] = axis == 0 ? se[k] / N_c : se[k] % N_c;
        __syncwarp();
        const int n = combine_by_key(key, sd, ord, tmp, sg, K);   // sums into sg
        const uint16_t *Wa = axis == 0 ? W_r : W_c;
        float *dWa = axis == 0 ? dW_r : dW_c;
        const int base = axis == 0 ? 0 : N_r;                    // row of the slot lists
        // a slot in each distinct row's list, all of the token's rows at once
        // (ord is free after combine_by_key); rcap = 0: no lists
        for (int u = lane; u < n; u += 32)
            ord[u] = rcap > 0 ? atomicAdd(&rcnt[base + key[u]], 1) : 0;
        __syncwarp();
        for (int u = 0; u < n; ++u) {
            const int r = key[u];
            const float ds = sg[u];
            uint4 wu[VPL];
            load_raw<VPL>(Wa + (size_t)r * D, wu, lane);
            axpy_bf16<VPL>(acc, ds, wu);
            const int slot = ord[u];
            if (slot < rcap) {
                if (lane == 0)
                    rslots[(size_t)(base + r) * rcap + slot] = make_int2(t, __float_as_int(ds));
            } else {
                red_row_bf16<VPL>(dWa + (size_t)r * D, ds, xu, lane);   // a full list
            }
        }
        __syncwarp();
    }
    float *dxr = dx + (size_t)t * D;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        float4 *p = reinterpret_cast<float4 *>(dxr + (size_t)(v * 32 + lane) * 8);
        p[0] = make_float4(acc[8 * v], acc[8 * v + 1], acc[8 * v + 2], acc[8 * v + 3]);
        p[1] = make_float4(acc[8 * v + 4], acc[8 * v + 5], acc[8 * v + 6], acc[8 * v + 7]);
    }
}

// Experts used by more than one task: seen / shared bitmaps over the N
// experts (both zeroed), one thread per task.  Ids outside [0, N) count as
// expert 0, as in the backward kernel.
__global__ void bwd_mark_kernel(const int32_t *__restrict__ idx, int64_t M, int N,
                                uint32_t *__restrict__ seen, uint32_t *__restrict__ shared_rows) {
    grid_dependency_wait();
    grid_dependents_launch();
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= M) return;
    int e = idx[i];
    if (e < 0 || e >= N) e = 0;
    const uint32_t bit = 1u << (e & 31);
    if (atomicOr(&seen[e >> 5], bit) & bit) atomicOr(&shared_rows[e >> 5], bit);
}

// The router rows' weight gradients from their slot lists: one warp per grid
// row (W_r rows, then W_c rows) sums ds * x_t over the row's (t, ds) pairs
// (four x rows in flight at a time) and adds the sum to its dW_r / dW_c row
// with one plain read-add-write: the warp owns the row, and the reductions of
// a full list's extra pairs finished with the previous kernel.
template <int VPL>
__global__ void __launch_bounds__(32 * kBwdWarps)
bwd_router_rows_kernel(const uint16_t *__restrict__ x, int L, int nrows, int N_r,
                       const int *__restrict__ rcnt, const int2 *__restrict__ rslots, int rcap,
                       float *__restrict__ dW_r, float *__restrict__ dW_c, int *status) {
    constexpr int D = 256 * VPL;
    constexpr int E = 8 * VPL;
    grid_dependency_wait();
    grid_dependents_launch();
    const int row = blockIdx.x * kBwdWarps + (int)(threadIdx.x >> 5);
    if (row >= nrows) return;                        // the same in every lane
    const unsigned lane = lane_id();
    const int cnt = min(rcnt[row], rcap);
    if (cnt <= 0) return;
    float acc[E];
#pragma unroll
    for (int c = 0; c < E; ++c) acc[c] = 0.f;
    const int2 *sl = rslots + (size_t)row * rcap;
    for (int s0 = 0; s0 < cnt; s0 += 32) {
        const int2 mine = s0 + (int)lane < cnt ? sl[s0 + lane] : make_int2(0, 0);
        const int m = min(32, cnt - s0);
        for (int j0 = 0; j0 < m; j0 += 4) {
            uint4 xu[4][VPL];
            float ds[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                int tq = __shfl_sync(0xffffffffu, mine.x, (j0 + q) & 31);
                ds[q] = __int_as_float(__shfl_sync(0xffffffffu, mine.y, (j0 + q) & 31));
                if (j0 + q >= m) ds[q] = 0.f;
                if (tq < 0 || tq >= L) {
                    set_status(status, OMNI_DEV_BAD_SCHEDULE);
                    tq = 0;
                    ds[q] = 0.f;
                }
                load_raw<VPL>(x + (size_t)tq * D, xu[q], lane);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) axpy_bf16<VPL>(acc, ds[q], xu[q]);
        }
    }
    float *dst = row < N_r ? dW_r + (size_t)row * D : dW_c + (size_t)(row - N_r) * D;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        float4 *p = reinterpret_cast<float4 *>(dst + (size_t)(v * 32 + lane) * 8);
        const float4 a = p[0], b = p[1];
        p[0] = make_float4(a.x + acc[8 * v], a.y + acc[8 * v + 1], a.z + acc[8 * v + 2],
                           a.w + acc[8 * v + 3]);
        p[1] = make_float4(b.x + acc[8 * v + 4], b.y + acc[8 * v + 5], b.z + acc[8 * v + 6],
                           b.w + acc[8 * v + 7]);
    }
}

template <int VPL>
cudaError_t launch_bwd_vpl(const uint16_t *x, const uint16_t *W, const uint16_t *V,
                           const uint16_t *W_r, const uint16_t *W_c, const Sizes &sz,
                           const int32_t *idx, const float *gate, const float *dy, float *dx,
                           float *dW, float *dV, float *dW_r, float *dW_c,
                           const uint32_t *shared_rows, int *rcnt, int2 *rslots, int rcap,
                           int *status, cudaStream_t st) {
    const size_t smem = (size_t)kBwdWarps * 6 * sz.K * 4;
    cudaError_t e = cudaFuncSetAttribute(routed_bwd_kernel<VPL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((sz.L + kBwdWarps - 1) / kBwdWarps);
    e = launch(routed_bwd_kernel<VPL>, dim3(grid), dim3(32 * kBwdWarps), smem, st, x, W, V,
                  W_r, W_c, sz.L, (int)sz.N, sz.N_c, sz.K, idx, gate, dy, dx, dW, dV, dW_r, dW_c,
                  shared_rows, rslots ? rcnt : nullptr, rslots, rslots ? rcap : 0, sz.N_r, status);
    if (e != cudaSuccess || !rslots) return e;
    const int nrows = sz.N_r + sz.N_c;
    return launch(bwd_router_rows_kernel<VPL>, dim3((unsigned)((nrows + kBwdWarps - 1) / kBwdWarps)),
                  dim3(32 * kBwdWarps), 0, st, x, sz.L, nrows, sz.N_r, (const int *)rcnt,
                  (const int2 *)rslots, rcap, dW_r, dW_c, status);
}

}  // namespace

cudaError_t launch_routed_bwd(const uint16_t *x, const uint16_t *W, const uint16_t *V,
                              const uint16_t *W_r, const uint16_t *W_c, const Sizes &sz,
                              const int32_t *idx, const float *gate, const float *dy, float *dx,
                              float *dW, float *dV, float *dW_r, float *dW_c, uint32_t *seen,
                              uint32_t *shared_rows, int *rcnt, int2 *rslots, int rcap,
                              int *status, cudaStream_t st) {
    if (seen && shared_rows) {
        const unsigned grid = (unsigned)((sz.M + 255) / 256);
        cudaError_t e = launch(bwd_mark_kernel, dim3(grid), dim3(256), 0, st, idx, (int64_t)sz.M,
                               (int)sz.N, seen, shared_rows);
        if (e != cudaSuccess) return e;
    } else {
        shared_rows = nullptr;
    }
    switch (sz.d / 256) {
#define OMNI_BCASE(n) \
        case n: return launch_bwd_vpl<n>(x, W, V, W_r, W_c, sz, idx, gate, dy, dx, dW, dV, dW_r, \
                                         dW_c, shared_rows, rcnt, rslots, rcap, status, st);
        OMNI_BCASE(1) OMNI_BCASE(2) OMNI_BCASE(3) OMNI_BCASE(4)
        OMNI_BCASE(5) OMNI_BCASE(6) OMNI_BCASE(7) OMNI_BCASE(8)
#undef OMNI_BCASE
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace omni

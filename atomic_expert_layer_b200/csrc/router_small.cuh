// router_small.cuh -- the streamed router projection for a handful of
// tokens (the small-batch projection kernel of the router stage call).
//
// "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale"
// (rainbus review page, method paragraph, step 2): s_r = x W_r and
// s_c = x W_c, with W_r / W_c stored as N_r / N_c rows of d.
#pragma once

#include "omni_common.cuh"

namespace omni {
namespace {

// ------------------------------------------------- few tokens
// The router's tile GEMM (router_gemm.cu) walks one 256-row tile through the
// whole K loop when a batch has a handful of tokens, which makes it
// latency-bound.  Then the
// projection is a streamed read of W_r and W_c: warp w of CTA b takes grid
// rows (kSmallRows * (kSmallWarps * b + w)) .. + kSmallRows - 1 (W_r rows,
// then W_c rows) and issues every load of them at once (lane l holds the
// 8-wide slices l, l + 32, ..., d <= 2048), the batch's x rows sit in shared
// memory, and each (row, token) dot product is reduced over the warp.  Only
// s is written; the axis selection then takes LogSoftmax itself.  Measured
// on B200 at d = 2048: faster than the tile GEMM at L = 1 (5.7 vs ~14 us).
// It serves the stand-alone projection for L <= 4; its slice width also
// bounds d in the fused decode step (d <= 32 * 8 * kSmallSlices).
constexpr int kSmallRows = 2;          // grid rows per warp
constexpr int kSmallWarps = 8;
constexpr int kSmallSlices = 8;        // 8-wide slices per lane: d <= 32 * 8 * 8

// The projection of one warp's kSmallRows grid rows g0, g0 + 1 (W_r rows,
// then W_c rows) with the L <= LM token rows staged in xs ([L][d / 8] uint4):
// every slice of the rows in flight at once, each (row, token) dot product
// reduced over the warp.  xs_ready() is called between issuing the row loads
// and reading xs (the caller's wait for its staging copies).
template <int LM, typename Ready>
__device__ __forceinline__ void small_rows_dot(const uint4 *xs, const uint16_t *__restrict__ W_r,
                                               const uint16_t *__restrict__ W_c, int L, int d,
                                               int N_r, int N_c, int g0, float *__restrict__ s_r,
                                               float *__restrict__ s_c, Ready xs_ready) {
    const int d8 = d >> 3;
    const unsigned lane = lane_id();
    const int ntot = N_r + N_c;
    // this warp's rows, every slice in flight at once
    uint4 wu[kSmallRows][kSmallSlices];
#pragma unroll
    for (int r = 0; r < kSmallRows; ++r) {
        const int g = g0 + r;                            // rows past the end: zeros, not written
        const uint4 *w4 = reinterpret_cast<const uint4 *>(
            g < N_r ? W_r + (size_t)g * d : W_c + (size_t)(g - N_r) * d);
#pragma unroll
        for (int i = 0; i < kSmallSlices; ++i) {
            const int c8 = (int)lane + 32 * i;
            wu[r][i] = c8 < d8 && g < ntot ? w4[c8] : make_uint4(0u, 0u, 0u, 0u);
        }
    }
    xs_ready();
    float acc[kSmallRows][LM];
#pragma unroll
    for (int r = 0; r < kSmallRows; ++r)
#pragma unroll
        for (int t = 0; t < LM; ++t) acc[r][t] = 0.f;
#pragma unroll
    for (int i = 0; i < kSmallSlices; ++i) {
        const int c8 = (int)lane + 32 * i;
        if (c8 < d8) {
            float wf[kSmallRows][8];
#pragma unroll
            for (int r = 0; r < kSmallRows; ++r) {
                const uint32_t w4[4] = {wu[r][i].x, wu[r][i].y, wu[r][i].z, wu[r][i].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    wf[r][2 * q] = __uint_as_float(w4[q] << 16);
                    wf[r][2 * q + 1] = __uint_as_float(w4[q] & 0xffff0000u);
                }
            }
#pragma unroll
            for (int t = 0; t < LM; ++t) {
                if (t < L) {
                    const uint4 u = xs[(size_t)t * d8 + c8];
                    const uint32_t x4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float xlo = __uint_as_float(x4[q] << 16);
                        const float xhi = __uint_as_float(x4[q] & 0xffff0000u);
#pragma unroll
                        for (int r = 0; r < kSmallRows; ++r) {
                            acc[r][t] = fmaf(xlo, wf[r][2 * q], acc[r][t]);
                            acc[r][t] = fmaf(xhi, wf[r][2 * q + 1], acc[r][t]);
                        }
                    }
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < kSmallRows; ++r) {
        const int g = g0 + r;
#pragma unroll
        for (int t = 0; t < LM; ++t) {
            if (t < L) {
                const float v = warp_sum(acc[r][t]);
                if (lane == 0 && g < ntot) {
                    if (g < N_r) s_r[(size_t)t * N_r + g] = v;
                    else s_c[(size_t)t * N_c + (g - N_r)] = v;
                }
            }
        }
    }
}

}  // namespace
}  // namespace omni

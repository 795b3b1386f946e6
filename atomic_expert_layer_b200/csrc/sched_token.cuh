// sched_token.cuh -- the per-token first step of the expert-centric schedule,
// shared by the schedule's own prepare kernel and by the router's merge
// kernel (which already holds a token's K experts and gates on chip when the
// whole routed forward runs).  When the schedule only groups the tasks (the
// routed forward), the order inside a token does not matter and the rank
// sort is skipped.
//
// "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale"
// (rainbus review page, method paragraph, step 3): the routing decisions
// become (token, expert, gate) tasks that are then sorted by expert and
// grouped by B consecutive experts.  For one token this step
//   - orders the token's K tasks by expert id and writes them at t*K + rank
//     (the input of the stable radix sort on the group id q = e / B, which
//     then yields the (q, token, expert) order),
//   - counts the tasks of every group,
//   - marks each expert in a bitmap; the first task to set a bit counts one
//     distinct expert,
//   - counts the first radix pass's digit per sort tile.
#pragma once

#include "omni_common.cuh"
#include "omni_internal.h"

namespace omni {

struct SchedPrep {          // where the per-token step writes (all in the workspace)
    int32_t *a_tok, *a_exp;
    float *a_gate;
    int32_t *counts;        // [G], zeroed by the caller
    uint32_t *bitmap;       // [ceil(N / 32)], zeroed; null: distinct experts not counted
    int32_t *num_distinct;  // [1], zeroed
    int32_t *hist0;         // [digits][ntiles] of the first pass, zeroed; null: no radix pass
    int64_t ntiles;
    uint32_t dmask0;        // digit mask of the first pass
    int B;
    int unordered;          // the tasks are only grouped (no radix pass follows): a token's
                            // tasks keep the routing's order, no rank sort by expert
};

__device__ __forceinline__ uint32_t sched_digit(int32_t e, int B, int shift, uint32_t dmask) {
    return ((uint32_t)(e / B) >> shift) & dmask;
}

// One warp, token t: e_s[0, K) are its experts (in range), gate_of(k) its gates.
template <typename GateOf>
__device__ __forceinline__ void sched_token(const SchedPrep &o, int t, int K, const int32_t *e_s,
                                            GateOf gate_of) {
    const unsigned lane = lane_id();
    const size_t row = (size_t)t * K;
    for (int u0 = 0; u0 < K; u0 += 32) {
        const int u = u0 + (int)lane;
        bool fresh = false;
        if (u < K) {
            const int32_t eu = e_s[u];
            int r = u;
            if (!o.unordered) {
                r = 0;
                for (int v = 0; v < K; ++v) {
                    const int32_t ev = e_s[v];
                    r += (ev < eu) | ((ev == eu) & (v < u));
                }
            }
            const size_t pos = row + r;
            o.a_tok[pos] = t;
            o.a_exp[pos] = eu;
            o.a_gate[pos] = gate_of(u);
            atomicAdd(&o.counts[eu / o.B], 1);
            if (o.bitmap) {
                const uint32_t bit = 1u << (eu & 31);
                fresh = (atomicOr(&o.bitmap[eu >> 5], bit) & bit) == 0u;   // first task of eu
            }
            if (o.hist0)
                atomicAdd(&o.hist0[(int64_t)sched_digit(eu, o.B, 0, o.dmask0) * o.ntiles +
                                   (int64_t)(pos / kSortTile)], 1);
        }
        const int nf = __popc(__ballot_sync(0xffffffffu, fresh));
        if (lane == 0 && nf) atomicAdd(o.num_distinct, nf);     // nf = 0 without a bitmap
    }
}

}  // namespace omni

// route.cuh — S1 for one token, shared by the routing kernel and the fused
// small-batch front kernel (both give bit-identical results).
//
// "mini-AGI PR #3", minagi/pool.py requested(): probs = softmax(logits), the
// top-k of probs, renormalised. Renormalising the top-k of a full softmax is a
// softmax over the k selected logits; that is what is computed, in fp32.
//
// One warp per token. Each lane keeps up to 8 of the E <= 256 logits in
// registers (expert lane + 32*i). k rounds of a warp argmax (butterfly
// shuffles) pick the experts in descending order; equal values go to the lower
// expert index, and -0.0 equals +0.0 (plain float compares on the given
// values, never on recomputed probabilities), so the indices are bit-exact.
#pragma once
#include "internal.h"

namespace moe {

constexpr int kRouteMaxPerLane = 8;  // E <= 256

// a beats b: larger value, or equal value and lower index
MOE_DEV bool route_beats(float va, int ia, float vb, int ib) { return va > vb || (va == vb && ia < ib); }

// The whole warp routes token `row` (E logits): lane j < k writes selection j
// to idx_out[j] / w_out[j]. Warp-uniform; every lane must call it.
MOE_DEV void route_one_token(const float* __restrict__ row, int E, int k, int32_t* __restrict__ idx_out,
                             float* __restrict__ w_out) {
    const int lane = threadIdx.x & 31;
    float v[kRouteMaxPerLane];
#pragma unroll
    for (int i = 0; i < kRouteMaxPerLane; ++i) {
        const int e = lane + 32 * i;
        v[i] = (e < E) ? __ldg(row + e) : -INFINITY;
    }
    uint32_t taken = 0;  // bit i: v[i] already selected
    // indices >= E never win: k <= E and a real -inf beats padding by index
    float sel_v = 0.f;
    int sel_i = 0;
    float top = 0.f;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 0x7FFFFFFF;
#pragma unroll
        for (int i = 0; i < kRouteMaxPerLane; ++i) {
            const int e = lane + 32 * i;
            if (!(taken >> i & 1u) && e < E && route_beats(v[i], e, bv, bi)) {
                bv = v[i];
                bi = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
            const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, off);
            if (route_beats(ov, oi, bv, bi)) {
                bv = ov;
                bi = oi;
            }
        }
        // every lane now holds the same winner
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (j == 0) top = bv;
        if (lane == j) {
            sel_v = bv;
            sel_i = bi;
        }
    }
    // softmax over the k selected (lane j < k holds selection j)
    const float ex = (lane < k) ? expf(sel_v - top) : 0.f;
    float s = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, off);
    if (lane < k) {
        idx_out[lane] = sel_i;
        w_out[lane] = ex / s;
    }
}

}  // namespace moe

// route.cuh — S1 for one token, shared by the routing kernel and the fused
// small-batch front kernel (both give bit-identical results).
//
// "mini-AGI PR #3", minagi/pool.py requested(): probs = softmax(logits), the
// top-k of probs, renormalised. Renormalising the top-k of a full softmax is a
// softmax over the k selected logits; that is what is computed, in fp32.
//
// One warp per token; see route_one_token below for the selection.
#pragma once
#include "internal.h"

namespace moe {

constexpr int kRouteMaxPerLane = 8;  // E <= 256

// Order-preserving map of a float to an unsigned key (NaN excluded): larger
// value <-> larger key; -0.0 is mapped like +0.0 so that the two compare equal.
MOE_DEV uint32_t route_key(float v) {
    uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
MOE_DEV float route_unkey(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// The whole warp routes token `row` (E logits): lane j < k writes selection j
// to idx_out[j] / w_out[j]. Warp-uniform; every lane must call it. Returns
// the first choice (warp-uniform); *kth_key (if given) gets the k-th selected
// value's key.
// Each round: every lane takes its best untaken logit (larger value, then
// lower expert index); one warp max-reduction of the keys gives the winning
// value and one min-reduction over the lanes holding it gives the lowest
// expert index among equal values.
// NK: keys a lane holds (E <= 32 NK); the routing kernel takes NK = 4 for E <= 128.
template <int NK = kRouteMaxPerLane>
MOE_DEV int route_one_token(const float* __restrict__ row, int E, int k, int32_t* __restrict__ idx_out,
                            float* __restrict__ w_out, uint32_t* kth_key = nullptr) {
    static_assert(NK >= 1 && NK <= kRouteMaxPerLane, "keys per lane");
    const int lane = threadIdx.x & 31;
    uint32_t key[NK];
#pragma unroll
    for (int i = 0; i < NK; ++i) {
        const int e = lane + 32 * i;
        key[i] = (e < E) ? route_key(__ldg(row + e)) : 0u;  // 0: below every real key (also -inf's)
    }
    uint32_t taken = 0;  // bit i: key[i] already selected (or padding)
#pragma unroll
    for (int i = 0; i < NK; ++i)
        if (lane + 32 * i >= E) taken |= 1u << i;
    float sel_v = 0.f;
    int sel_i = 0;
    float top = 0.f;
    int first = 0;
    for (int j = 0; j < k; ++j) {
        uint32_t bk = 0;
        int bi = 0x7FFFFFFF;
#pragma unroll
        for (int i = 0; i < NK; ++i)
            if (!(taken >> i & 1u) && (key[i] > bk || bi == 0x7FFFFFFF)) {  // first untaken, then strictly larger
                bk = key[i];
                bi = lane + 32 * i;
            }
        const uint32_t kmax = __reduce_max_sync(0xFFFFFFFFu, bk);
        const int wi = int(__reduce_min_sync(0xFFFFFFFFu, (bi != 0x7FFFFFFF && bk == kmax) ? uint32_t(bi) : 0xFFFFFFFFu));
        if ((wi & 31) == lane) taken |= 1u << (wi >> 5);
        const float wv = route_unkey(kmax);
        if (kth_key && j == k - 1) *kth_key = kmax;
        if (j == 0) {
            top = wv;
            first = wi;
        }
        if (lane == j) {
            sel_v = wv;
            sel_i = wi;
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
    return first;
}

}  // namespace moe

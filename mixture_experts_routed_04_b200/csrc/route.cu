// route.cu — S1: top-k routing with a softmax over the selected logits.
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
#include "internal.h"

namespace moe {

namespace {

constexpr int kMaxPerLane = 8;  // E <= 256

// a beats b: larger value, or equal value and lower index
MOE_DEV bool beats(float va, int ia, float vb, int ib) { return va > vb || (va == vb && ia < ib); }

__global__ void __launch_bounds__(256) route_topk_softmax_kernel(const float* __restrict__ logits, int T, int E,
                                                                 int k, int32_t* __restrict__ topk_idx,
                                                                 float* __restrict__ topk_w) {
    griddep_wait();
    griddep_launch();
    const int lane = threadIdx.x & 31;
    const int warps_per_block = blockDim.x >> 5;
    const int64_t t = int64_t(blockIdx.x) * warps_per_block + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* row = logits + t * E;

    float v[kMaxPerLane];
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
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
        for (int i = 0; i < kMaxPerLane; ++i) {
            const int e = lane + 32 * i;
            if (!(taken >> i & 1u) && e < E && beats(v[i], e, bv, bi)) {
                bv = v[i];
                bi = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
            const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, off);
            if (beats(ov, oi, bv, bi)) {
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
        topk_idx[t * k + lane] = sel_i;
        topk_w[t * k + lane] = ex / s;
    }
}

}  // namespace

cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* topk_idx, float* topk_w,
                         cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    const int threads = 256, wpb = threads / 32;
    const int blocks = (T + wpb - 1) / wpb;
    {
        ProfScope prof_(MOE_K_ROUTE, stream);
        const cudaError_t le = launch_pdl(use_pdl(T), route_topk_softmax_kernel, dim3(blocks), dim3(threads), 0,
                                          stream, logits, T, E, k, topk_idx, topk_w);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe

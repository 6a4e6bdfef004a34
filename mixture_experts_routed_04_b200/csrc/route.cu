// route.cu — S1: top-k routing with a softmax over the selected logits.
//
// "mini-AGI PR #3", minagi/pool.py requested(): probs = softmax(logits), the
// top-k of probs, renormalised. Renormalising the top-k of a full softmax is a
// softmax over the k selected logits; that is what is computed, in fp32.
//
// One warp per token (route_one_token in route.cuh). Each lane keeps up to 8 of
// the E <= 256 logits as order-preserving integer keys (expert lane + 32*i).
// k rounds pick the experts in descending order: every lane offers its best
// untaken key, one warp max-reduction gives the winning value and one
// min-reduction over the lanes holding it the lowest expert index, so equal
// values go to the lower index and -0.0 equals +0.0 (the keys are built from
// the given values, never from recomputed probabilities): the indices are
// bit-exact.
#include "route.cuh"

namespace moe {

namespace {

// One warp per token (route_one_token, shared with the fused small-batch front kernel).
__global__ void __launch_bounds__(256) route_topk_softmax_kernel(const float* __restrict__ logits, int T, int E,
                                                                 int k, int32_t* __restrict__ topk_idx,
                                                                 float* __restrict__ topk_w) {
    griddep_wait();
    griddep_launch();
    const int warps_per_block = blockDim.x >> 5;
    const int64_t t = int64_t(blockIdx.x) * warps_per_block + (threadIdx.x >> 5);
    if (t >= T) return;
    route_one_token(logits + t * E, E, k, topk_idx + t * k, topk_w + t * k);
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

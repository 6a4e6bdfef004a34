// schedule.cu — K3: the tile schedule and per-expert variant choice as its own
// one-block kernel for moe_expert_ffn (moe_forward computes it inside the fused
// small-batch front kernel, or inside the permutation's scan for larger
// batches). The schedule itself is schedule_block.
#include "schedule.cuh"

namespace moe {

namespace {

// One block of 512 threads; thread e owns expert e (Etot <= 257).
__global__ void __launch_bounds__(512) schedule_kernel(const int32_t* __restrict__ offsets, int Etot, int variant,
                                                       int stream_max, int32_t* __restrict__ tile_base,
                                                       int32_t* __restrict__ stream_list,
                                                       int32_t* __restrict__ n_stream, uint32_t* err) {
    __shared__ int sums[3][16];
    griddep_wait();
    griddep_launch();
    const int e = threadIdx.x;
    int kept = 0;
    if (e < Etot) {
        kept = offsets[e + 1] - offsets[e];
        if (kept < 0) {
            set_error(err, MOE_DEVERR_BOUNDS);
            kept = 0;
        }
    }
    schedule_block(kept, Etot, variant, stream_max, sums, tile_base, stream_list, n_stream);
}

}  // namespace

cudaError_t launch_schedule(const Dims& D, const int32_t* offsets, int32_t* tile_base, int32_t* stream_list,
                            int32_t* n_stream, uint32_t* err, cudaStream_t s) {
    {
        ProfScope prof_(MOE_K_SCHEDULE, s);
        const cudaError_t le = launch_pdl(use_pdl(D.T), schedule_kernel, dim3(1), dim3(512), 0, s, offsets, D.Etot,
                                          D.variant, D.stream_max_rows, tile_base, stream_list, n_stream, err);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe

// schedule.cu — K3: the tile schedule and per-expert variant choice as its own
// one-block kernel (batches of more than 64 tokens; smaller batches compute it
// inside the fused front kernel). The schedule itself is schedule_block; this
// kernel also writes the claim order of the tcgen05 GEMMs' units.
//
// Claim order. A unit is (expert e, n-tile n, M-tile m); the units of one
// (e, n) — a "group" — share one weight tile (K x 256 columns). The first
// unit of a group to run (its leader, m = 0) streams that tile from HBM; the
// others find it in L2. Claimed in the natural order, a large expert's units
// all start together and wait on the one leader's HBM stream (an L2 miss in
// flight serves them all), so few distinct weight streams are in flight and
// HBM idles. Here groups are cut into chunks of `chunk` consecutive groups and
// the units are claimed as
//     leaders of chunk 0, leaders of chunk 1, followers of chunk 0,
//     leaders of chunk 2, followers of chunk 1, ...
// so every follower is claimed at least `chunk` units after its leader, while
// the next chunk's leaders keep many weight streams in flight. chunk = 0 keeps
// the natural order. Which CTA computes a unit, and when, does not change its
// result.
#include "schedule.cuh"

namespace moe {

namespace {

// One block of 512 threads; thread e owns expert e (Etot <= 257); the
// schedule itself is schedule_block (shared with the fused front kernel).
// With units_a non-null it then writes the claim orders of the two GEMMs
// (nt_a and nt_b n-tiles per M-tile; M-tiles of `sub` x 128 rows).
__global__ void __launch_bounds__(512) schedule_kernel(const int32_t* __restrict__ offsets, int Etot, int variant,
                                                       int stream_max, int32_t* __restrict__ tile_base,
                                                       int32_t* __restrict__ stream_list,
                                                       int32_t* __restrict__ n_stream, uint32_t* err, int sub,
                                                       int nt_a, int nt_b, int chunk, long long* units_a,
                                                       long long* units_b) {
    __shared__ int sums[3][16];
    __shared__ int s_tb[kMaxE + 2], s_ne[kMaxE + 2];
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
    if (units_a) unit_orders_block(tile_base, Etot, sub, nt_a, nt_b, chunk, units_a, units_b, s_tb, s_ne, sums);
}

}  // namespace

cudaError_t launch_schedule(const Dims& D, const int32_t* offsets, int32_t* tile_base, int32_t* stream_list,
                            int32_t* n_stream, uint32_t* err, const UnitOrder& order, cudaStream_t s) {
    int smax = D.stream_max_rows;
    {
        ProfScope prof_(MOE_K_SCHEDULE, s);
        const cudaError_t le =
            launch_pdl(use_pdl(D.T), schedule_kernel, dim3(1), dim3(512), 0, s, offsets, D.Etot, D.variant, smax,
                       tile_base, stream_list, n_stream, err, order.sub, order.nt_a, order.nt_b, order.chunk,
                       order.units_a, order.units_b);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe

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

// Exclusive prefix over experts of "has at least one M-tile", into ne[0..Etot].
MOE_DEV void nonempty_prefix(const int* tb, int Etot, int* ne, int* wsum) {
    const int e = threadIdx.x, lane = e & 31, w = e >> 5;
    const int f = (e < Etot && tb[e + 1] > tb[e]) ? 1 : 0;
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, f);
    uint32_t lt;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt));
    if (lane == 31) wsum[w] = __popc(bal);
    __syncthreads();
    int base = 0;
    for (int i = 0; i < w; ++i) base += wsum[i];
    if (e <= Etot) ne[e] = base + __popc(bal & lt);
    __syncthreads();
}

// Positions of every unit of one GEMM (nt n-tiles per M-tile) in claim order;
// writes units[pos] = (e << 48 | n << 32 | m). Block-wide.
MOE_DEV void unit_order_list(const int* tb, const int* ne, int Etot, int nt, int chunk, long long* units) {
    const int G = Etot * nt;
    auto mt = [&](int e) { return tb[e + 1] - tb[e]; };
    // units before group g in the natural order, and non-empty groups (leaders) before g
    auto U = [&](int g) {
        if (g >= G) return tb[Etot] * nt;
        const int e = g / nt, n = g - e * nt;
        return tb[e] * nt + n * mt(e);
    };
    auto NL = [&](int g) {
        if (g >= G) return ne[Etot] * nt;
        const int e = g / nt, n = g - e * nt;
        return ne[e] * nt + (mt(e) > 0 ? n : 0);
    };
    auto FB = [&](int g) { return U(g) - NL(g); };  // followers before group g
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        const int e = g / nt, n = g - e * nt, m_e = mt(e);
        if (m_e == 0) continue;
        const unsigned long long key = (static_cast<unsigned long long>(e) << 48) |
                                       (static_cast<unsigned long long>(n) << 32);
        if (chunk <= 0) {
            const int u0 = U(g);
            for (int m = 0; m < m_e; ++m) units[u0 + m] = static_cast<long long>(key | unsigned(m));
            continue;
        }
        const int c = g / chunk, g0 = c * chunk;
        const int startL = c == 0 ? 0 : NL(g0) + FB(g0 - chunk);
        const int startF = NL(g0 + 2 * chunk) + FB(g0);
        units[startL + NL(g) - NL(g0)] = static_cast<long long>(key);
        const int f0 = startF + FB(g) - FB(g0) - 1;
        for (int m = 1; m < m_e; ++m) units[f0 + m] = static_cast<long long>(key | unsigned(m));
    }
}

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
    if (!units_a) return;
    __syncthreads();  // this block's tile_base writes are visible to the block
    const int32_t* tb = tile_base + (sub == 2 ? Etot + 1 : 0);
    if (e <= Etot) s_tb[e] = tb[e];
    __syncthreads();
    nonempty_prefix(s_tb, Etot, s_ne, &sums[0][0]);
    unit_order_list(s_tb, s_ne, Etot, nt_a, chunk, units_a);
    unit_order_list(s_tb, s_ne, Etot, nt_b, chunk, units_b);
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

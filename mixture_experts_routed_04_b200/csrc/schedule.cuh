// schedule.cuh — K3, the tile schedule and variant choice, shared by the
// schedule kernel and the fused small-batch front kernel.
#pragma once
#include "internal.h"

namespace moe {

// One block of at least Etot threads (at most 512); thread e owns expert e and
// passes its kept row count (0 for e >= Etot). Writes:
//   tile_base[0 .. Etot]           exclusive prefix of 128-row tiles per expert
//   tile_base[Etot+1 .. 2*Etot+1]  that of 256-row tiles (Q4G32 and SM-pair units)
//   stream_list[0 .. n)            experts taken by the streaming kernels
//   n_stream[0] = n; n_stream[1] = n_stream[2] = 0 (unit counters of the GEMMs)
// Every thread of the block must call it (it synchronises the block).
MOE_DEV void schedule_block(int kept, int Etot, int variant, int stream_max, int (*sums)[16],
                            int32_t* __restrict__ tile_base, int32_t* __restrict__ stream_list,
                            int32_t* __restrict__ n_stream) {
    const int e = threadIdx.x, lane = e & 31, w = e >> 5;
    const int is_stream =
        (kept > 0 && (variant == MOE_VARIANT_STREAM || (variant == MOE_VARIANT_AUTO && kept <= stream_max))) ? 1 : 0;
    const int tiles = (kept > 0 && !is_stream) ? (kept + kTileM - 1) / kTileM : 0;
    const int tiles2 = (tiles + 1) >> 1;
    int it = tiles, is = is_stream, i2 = tiles2;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int a = __shfl_up_sync(0xFFFFFFFFu, it, off);
        const int b = __shfl_up_sync(0xFFFFFFFFu, is, off);
        const int c = __shfl_up_sync(0xFFFFFFFFu, i2, off);
        if (lane >= off) {
            it += a;
            is += b;
            i2 += c;
        }
    }
    if (lane == 31) {
        sums[0][w] = it;
        sums[1][w] = is;
        sums[2][w] = i2;
    }
    __syncthreads();
    int bt = 0, bs = 0, b2 = 0, tt = 0, ts = 0, t2 = 0;
    const int nw = int(blockDim.x >> 5);
    for (int i = 0; i < nw; ++i) {
        if (i < w) {
            bt += sums[0][i];
            bs += sums[1][i];
            b2 += sums[2][i];
        }
        tt += sums[0][i];
        ts += sums[1][i];
        t2 += sums[2][i];
    }
    if (e < Etot) {
        tile_base[e] = bt + it - tiles;
        tile_base[Etot + 1 + e] = b2 + i2 - tiles2;
    }
    if (is_stream) stream_list[bs + is - 1] = e;
    if (e == 0) {
        tile_base[Etot] = tt;
        tile_base[2 * Etot + 1] = t2;
        n_stream[0] = ts;
        n_stream[1] = 0;  // unit counters of the two tcgen05 GEMMs (claimed with atomicAdd)
        n_stream[2] = 0;
    }
}

}  // namespace moe

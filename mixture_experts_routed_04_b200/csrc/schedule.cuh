// schedule.cuh — K3, the tile schedule and variant choice, shared by the
// schedule kernel and the fused small-batch front kernel.
#pragma once
#include "internal.h"

namespace moe {

// One block of 512 threads; thread e owns expert e (Etot <= 257) and passes its
// kept row count (0 for e >= Etot). Writes:
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
    for (int i = 0; i < 16; ++i) {
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

// After schedule_block (every thread of the 512-thread block): the claim orders
// of the two tile GEMMs from the tile prefix it wrote (see schedule.cu).
MOE_DEV void unit_orders_block(const int32_t* tile_base, int Etot, int sub, int nt_a, int nt_b, int chunk,
                               long long* units_a, long long* units_b, int* s_tb, int* s_ne, int (*sums)[16]) {
    __syncthreads();  // this block's tile_base writes are visible to the block
    const int e = threadIdx.x;
    const int32_t* tb = tile_base + (sub == 2 ? Etot + 1 : 0);
    if (e <= Etot) s_tb[e] = tb[e];
    __syncthreads();
    nonempty_prefix(s_tb, Etot, s_ne, &sums[0][0]);
    unit_order_list(s_tb, s_ne, Etot, nt_a, chunk, units_a);
    unit_order_list(s_tb, s_ne, Etot, nt_b, chunk, units_b);
}

}  // namespace moe

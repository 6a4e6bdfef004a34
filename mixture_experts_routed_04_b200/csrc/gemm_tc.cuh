// gemm_tc.cuh — pieces shared by the two tcgen05 grouped GEMM kernels (one SM
// per 128-row tile in gemm_tc.cu, SM pairs on 256-row tiles in gemm_pair.cu):
// tile constants, kernel parameters, work-unit decoding, the fused SwiGLU, the
// shared-memory unit ring and the epilogue of one 128-row accumulator.
#pragma once

#include "schedule.cuh"

namespace moe {

namespace tc {

constexpr int BM = 128, BK = 64, BN = 256;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_CHUNK = 64 * BK * 2;  // one 64(N) x 64(K) box, 8 KB
constexpr int B_BYTES = 4 * B_CHUNK;  // 32 KB (256 N x 64 K, 2-byte elements)
constexpr int P_BYTES = BN * BK / 2;  // Q4G32 nibbles of 256 rows x 64 K: 8 KB
constexpr int S_BYTES = 2 * BN * 2;   // two scale groups x 256 rows, fp16: 1 KB
constexpr int TMEM_COLS = 512;

struct GemmParams {
    int K;        // reduction length (multiple of 64)
    int n_out;    // output width
    int n_tiles;  // output tiles per M-tile
    int E;        // routed experts; index E is the shared expert
    int Etot;
    int32_t* unit_counter;     // next unit to claim (zeroed by the schedule kernel)
    const int32_t* tile_base;  // [Etot+1] exclusive prefix of M-tiles
    const int32_t* offsets;    // [Etot+1] row offsets
    uint16_t* out;             // [rows, n_out] fp16 (h or y)
    const int32_t* sorted_pair;
    const float* topk_w;
    float limit;
    uint32_t* err;
    uint64_t wait_ns;
    // Rows gathered inside the gate/up GEMM (GATHER kernels): A row r of expert
    // rows is x[sorted_token[r]], x [T, d] bf16.
    const uint16_t* x;
    const int32_t* sorted_token;
    int T;
};

struct Unit {
    int e, m, n, row0, rows;
};

// p.tile_base counts units of SUB x 128 rows. Units are claimed expert by
// expert, each n-tile's M-tiles in turn, so the M-tiles sharing a weight tile
// run together and read it from L2 after the first. (Claim orders that ran an
// n-tile's first M-tile a chunk of 16 to 64 groups ahead of the others, to put
// more distinct weight streams in flight, measured 2-12% slower on B200.)
template <int SUB>
MOE_DEV Unit decode_unit(int u, const GemmParams& p, int nt) {
    Unit U;
    const int g = u / nt;  // global M-tile index
    int lo = 0, hi = p.Etot;      // tile_base[lo] <= g < tile_base[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(p.tile_base + mid) <= g) lo = mid;
        else hi = mid;
    }
    U.e = lo;
    const int tb = __ldg(p.tile_base + lo);
    const int mt = __ldg(p.tile_base + lo + 1) - tb;
    const int local = u - tb * nt;
    U.n = local / mt;
    U.m = local - U.n * mt;
    const int off = __ldg(p.offsets + U.e);
    const int kept = __ldg(p.offsets + U.e + 1) - off;
    U.row0 = off + U.m * (SUB * BM);
    U.rows = min(SUB * BM, kept - U.m * (SUB * BM));
    return U;
}

MOE_DEV float swiglu(float g, float u, float L) {
    if (L > 0.f) {
        g = fminf(fmaxf(g, -L), L);
        u = fminf(fmaxf(u, -L), L);
    }
    // __expf / __fdividef: relative error ~1e-6, far below the fp16 rounding
    // of h that follows (the accurate forms cost ~5% of the gate/up GEMM).
    return __fdividef(g, 1.0f + __expf(-g)) * u;
}

// ---------------------------------------------------------------- unit ring
// Work is claimed dynamically: the producer warp takes the next unit with an
// atomic counter and publishes it in a shared-memory ring that the MMA,
// epilogue and transform warps read in order. A CTA that draws slow
// (DRAM-bound) units therefore takes fewer of them and every SM finishes
// together. Which CTA computes a unit does not change its result.
constexpr int UR = 8;  // ring depth; the producer runs at most ~2 units ahead of the epilogue

// Producer: claim and publish the next unit (-1 when none is left). Returns
// false if the bounded wait gave up. Warp-uniform.
MOE_DEV bool ring_publish(int& u, int& slot, uint32_t& phase, int* counter, int total, volatile int* ring,
                          uint64_t* ufull, uint64_t* uempty, volatile int* abort_flag, uint32_t* err, uint64_t ns) {
    const int lane = threadIdx.x & 31;
    int ok = 1;
    if (lane == 0) ok = mbar_wait_bounded(uempty + slot, phase ^ 1u, abort_flag, err, ns);
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    if (!ok) return false;
    int v = 0;
    if (lane == 0) {
        v = atomicAdd(counter, 1);
        if (v >= total) v = -1;
        ring[slot] = v;
        mbar_arrive(ufull + slot);
    }
    u = __shfl_sync(0xFFFFFFFFu, v, 0);
    if (++slot == UR) {
        slot = 0;
        phase ^= 1u;
    }
    return true;
}

// Reader: the next published unit (-1: done). Returns false if the wait gave up.
MOE_DEV bool ring_read(int& u, int& slot, uint32_t& phase, volatile int* ring, uint64_t* ufull, uint64_t* uempty,
                       volatile int* abort_flag, uint32_t* err, uint64_t ns) {
    const int lane = threadIdx.x & 31;
    int ok = 1;
    if (lane == 0) ok = mbar_wait_bounded(ufull + slot, phase, abort_flag, err, ns);
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    if (!ok) return false;
    int v = 0;
    if (lane == 0) {
        v = ring[slot];
        mbar_arrive(uempty + slot);
    }
    u = __shfl_sync(0xFFFFFFFFu, v, 0);
    if (++slot == UR) {
        slot = 0;
        phase ^= 1u;
    }
    return true;
}

// Epilogue of one accumulator of up to 128 rows x 256 columns: warp quadrant q
// reads TMEM lanes 32q..32q+31 from column address tb (lane field included) and
// writes its rows (the first `rows` of the tile) of p.out for output tile n.
// Row r of the tile sits in lane r (M=128, and each CTA's half of an SM-pair
// M=256 tile); with m64 (a tile computed at M=64), in lane 32*(r/16) + r%16.
//   MODE 0: columns 0-127 gate, 128-255 up -> h = SwiGLU, 128 output columns.
//   MODE 1: 256 columns scaled by the pair's gate weight (1 for the shared expert).
// Values outside fp16's range set range_bad.
template <int MODE>
MOE_DEV void epilogue_tile(uint32_t tb, int n, int64_t row0, int rows, bool m64, int q, int lane,
                           const GemmParams& p, bool& range_bad) {
    const int rit = m64 ? q * 16 + lane : q * 32 + lane;
    const bool valid = (!m64 || lane < 16) && rit < rows;
    const int64_t row = row0 + rit;
    if (MODE == 0) {
        constexpr int hw = 128;
#pragma unroll 1
        for (int c = 0; c < hw / 32; ++c) {
            uint32_t g[32], v[32];
            tmem_ld_32x32b_x32(tb + c * 32, g);
            tmem_ld_32x32b_x32(tb + hw + c * 32, v);
            tmem_ld_wait();
            const int col = n * hw + c * 32;
            if (valid && col < p.n_out) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float h0 = swiglu(__uint_as_float(g[2 * i]), __uint_as_float(v[2 * i]), p.limit);
                    const float h1 = swiglu(__uint_as_float(g[2 * i + 1]), __uint_as_float(v[2 * i + 1]), p.limit);
                    range_bad |= !(f16_range_ok(h0) && f16_range_ok(h1));
                    pk[i] = pack_f16x2(h0, h1);
                }
                uint4* dst = reinterpret_cast<uint4*>(p.out + row * p.n_out + col);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
        }
    } else {
        float w = 0.f;
        if (valid) {
            const int sp = __ldg(p.sorted_pair + row);
            w = sp >= 0 ? __ldg(p.topk_w + sp) : 1.0f;
        }
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tb + c * 32, v);
            tmem_ld_wait();
            const int col = n * BN + c * 32;
            if (valid && col < p.n_out) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float y0 = w * __uint_as_float(v[2 * i]);
                    const float y1 = w * __uint_as_float(v[2 * i + 1]);
                    range_bad |= !(f16_range_ok(y0) && f16_range_ok(y1));
                    pk[i] = pack_f16x2(y0, y1);
                }
                uint4* dst = reinterpret_cast<uint4*>(p.out + row * p.n_out + col);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
        }
    }
}

// ---- host side (gemm_tc.cu): tensor maps
// A operand: rows x K 2-byte elements, row-major; box 64 (K) x 128 (rows), 128-byte swizzle.
bool map_rows(CUtensorMap* m, const void* base, int64_t rows, int K);
// bf16/fp16 B operand [nexp, K, N]; one copy brings `chunks` 64-column boxes of 64 K-rows.
bool map_weights(CUtensorMap* m, const void* base, int nexp, int K, int N, int chunks);
// The SM-pair kernels (gemm_pair.cu): MODE 0 bf16 gate/up (B0/B1 = W_gate/W_up,
// S0/S1 = the shared expert's), MODE 1 fp16 W_down (B0, S0); maps of 2 chunks.
template <int MODE>
cudaError_t launch_gemm_pair(const CUtensorMap& A, const CUtensorMap& B0, const CUtensorMap& B1, const CUtensorMap& S0,
                             const CUtensorMap& S1, const GemmParams& p, bool pdl, cudaStream_t s);

}  // namespace tc

}  // namespace moe

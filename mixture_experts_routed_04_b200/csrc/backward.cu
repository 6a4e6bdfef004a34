// backward.cu — gradients of the routed expert FFN (and of the routing weights)
// for an upstream gradient dout = dL/dout, on the 5th-generation tensor cores.
//
// "mini-AGI PR #3", tests/test_dispatch.py: the expert weights w1, w3, w2
// (gate, up, down) receive the same gradients on every dispatch path; the
// layer trains through this path. With y = swiglu(x Wg, x Wu) Wd and
// out[t] = sum_j w[t,j] y[t,j], a kept pair's expert sees dy = w * dout[t]:
//   dh = dy Wd^T; (dg, du) = clamped-SwiGLU backward; dx_row = dg Wg^T + du Wu^T
//   dWd = h^T dy;  dWg = x^T dg;  dWu = x^T du
//   d w[t,j] = <dout[t], y[t,j]> = <h, dout[t] Wd^T>;  dlogits through the
//   softmax over the k selected logits.
//
// Row space: every expert's rows are padded to a multiple of 64 with zero
// rows (poff[e] = padded offset), so the weight gradients, which contract
// over an expert's rows, run whole 64-row k-blocks. Launches (one stream):
//   bwd_schedule      padded offsets, tile prefixes, unit counters
//   bwd_gather        xg = x rows (bf16 and fp16), dog = dout rows (fp16), zero padding rows
//   GEMM GU           x [Wg|Wu] -> g, u, w h (fp16)
//   GEMM DH           dout_rows Wd^T -> dh = w dhu -> dg, du (bf16 and fp16); <h, dhu> with
//                     h = silu(clamp g) clamp u recomputed from the stored g, u
//   GEMM DX           [dg|du] [Wg|Wu]^T -> dx rows (fp16, real row order)
//   GEMM WG x3        dWd = (w h)^T dout_rows; dWg = xg^T dg; dWu = xg^T du (A read
//                     N-major straight from the row buffers: no transposed copy)
//   zero_untouched    zero weight gradients of experts without rows
//   combine           dx[t] = sum of its pairs' dx rows (+ shared)
//   dw_reduce         d topk_w[p] = sum over n-tiles of <h, dhu>
//   route_backward    dlogits (optional)
// Operands: GU and DX multiply the bf16 gate/up weights, so x and dg, du enter
// them as bf16; DH multiplies the fp16 copy of W_down (prepared once, as for the
// forward) by fp16 dout rows; the weight gradients multiply fp16 activations.
// fp32 accumulation (TMEM) throughout. (All-bf16 operands measured 8x larger
// weight-gradient errors: rounding dout and dg to 8 significant bits.) The GEMM kernel is the
// forward kernel's structure (TMA producer warp, one-thread MMA issuer,
// four epilogue warps, unit ring, bounded waits) with per-mode loads and
// epilogues; A is K-major (rows) or, for the weight gradients, N-major (the
// row buffers read as [K = rows, M]); B K-major (weights read transposed: DH,
// DX) or N-major (weights as stored: GU; activations: WG). The weight-gradient
// tiles (fp32) go out through shared memory as whole 128-byte row segments.
#include "gemm_tc.cuh"

namespace moe {

namespace bwd {

using tc::A_BYTES;
using tc::B_BYTES;
using tc::B_CHUNK;
using tc::BK;
using tc::BM;
using tc::BN;
using tc::TMEM_COLS;
using tc::UR;

enum { GU = 0, DH = 1, DX = 2, WG = 3 };

constexpr int kStages = 4;
constexpr int kStageBytes = A_BYTES + B_BYTES;
// Eight epilogue warps, two per 32-lane TMEM quadrant, each taking every other
// 32-column chunk: the epilogues load and store per row (g, u, dg, du, dx, the
// gradient tiles), and four warps left the MMAs waiting on them.
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kStageOut = kEpiWarps * 32 * 32 * 4;  // WG: one 32 x 32 fp32 block per epilogue warp
// + barriers and unit ring (512), padding so the staging blocks are 1024-byte aligned
// (the 128-byte-swizzled boxes of the TMA stores)
constexpr int kSmem = 1024 + kStages * kStageBytes + 1024 + kStageOut;
constexpr int kUnitReaders = 1 + kEpiWarps;
constexpr int kPad = 64;  // rows of an expert are padded to a multiple of this

struct Params {
    int K;        // reduction length of the row GEMMs (GU, DH: d; DX: 2f)
    int n_tiles;  // output tiles per M-tile
    int E, Etot;
    int d, f;
    int64_t rp;                // padded rows allocated
    int32_t* unit_counter;
    const int32_t* tile_base;  // [Etot+1] prefix of 128-row M-tiles over padded rows
    const int32_t* poff;       // [Etot+1] padded row offsets
    const int32_t* wbase;      // [Etot+1] prefix of experts with rows (WG units)
    const int32_t* offsets;    // [Etot+1] row offsets
    const int32_t* sorted_pair;
    const float* topk_w;
    float limit;
    // outputs
    uint16_t* gu;      // [rp, 2f] fp16 g then u (outside the clamp: +-next fp16 above L)
    uint16_t* hw;      // [rp, f] fp16, w * h
    uint16_t* dgu;     // [rp, 2f] bf16, dg then du (operand of DX)
    uint16_t* dgu16;   // [rp, 2f] fp16, the same (operand of the weight gradients)
    uint16_t* dxr;     // [rows, d] fp16, real row order
    float* dwp;        // [rows, 2 x n_tiles of DH] partial <h, dhu> (per DH n-tile, per epilogue half)
    float* dw;         // WG: routed experts' gradient [E, M, N]
    float* sdw;        // WG: the shared expert's [M, N]
    int M, N;          // WG output dims
    uint32_t* err;
    uint64_t wait_ns;
};

struct Unit {
    int e, m, n;
    int row0;  // padded row of the tile's first row (row modes) / first M row (WG)
    int rows;  // rows of the tile inside the expert's padded rows (row modes) / M rows (WG)
    int kb;    // k-blocks
};

template <int MODE>
MOE_DEV Unit decode(int u, const Params& p) {
    Unit U;
    if (MODE == WG) {
        const int mt = (p.M + BM - 1) / BM, nt = (p.N + BN - 1) / BN;
        const int g = u / (mt * nt);
        int lo = 0, hi = p.Etot;  // wbase[lo] <= g < wbase[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(p.wbase + mid) <= g) lo = mid;
            else hi = mid;
        }
        U.e = lo;
        const int local = u - g * (mt * nt);
        U.n = local / mt;
        U.m = local - U.n * mt;
        U.row0 = U.m * BM;
        U.rows = min(BM, p.M - U.row0);
        U.kb = (__ldg(p.poff + lo + 1) - __ldg(p.poff + lo)) / BK;
    } else {
        const int nt = p.n_tiles;
        const int g = u / nt;
        int lo = 0, hi = p.Etot;
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
        const int po = __ldg(p.poff + lo);
        const int rpad = __ldg(p.poff + lo + 1) - po;
        U.row0 = po + U.m * BM;
        U.rows = min(BM, rpad - U.m * BM);
        U.kb = p.K / BK;
    }
    return U;
}

MOE_DEV float silu_f(float z, float& s) {
    s = __fdividef(1.0f, 1.0f + __expf(-z));
    return z * s;
}

// Epilogue of one unit: warp quadrant q holds tile rows 32q..32q+31 (lane = row).
// The fp16 store of a pre-activation for the SwiGLU backward: v itself inside
// [-L, L] (rounding never leaves it: L is an fp16 value and rounding is
// monotone), else the next fp16 beyond +-L, so the backward clamps it back to
// +-L and sees it outside the range exactly when v was.
MOE_DEV float clamp_code(float v, float L) {
    if (!(L > 0.f) || fabsf(v) <= L) return v;
    const float beyond = f16_lo((pack_f16x2(L, 0.f) & 0xFFFFu) + 1u);  // L > 0: one fp16 step above
    return v > 0.f ? beyond : -beyond;
}

// Row modes: the padded row this thread writes, its real row (-1 for padding
// or past the tile) and the pair's gate weight (1 for the shared expert, 0 for
// padding). Loaded before the accumulator is waited for, so the dependent
// loads overlap the unit's MMAs.
struct RowInfo {
    int real;
    float w;
};
MOE_DEV RowInfo row_info(const Unit& U, int q, int lane, const Params& p) {
    RowInfo r{-1, 0.f};
    const int rit = q * 32 + lane;
    if (rit >= U.rows) return r;
    const int j = U.row0 + rit - __ldg(p.poff + U.e);
    const int off = __ldg(p.offsets + U.e);
    if (j < __ldg(p.offsets + U.e + 1) - off) {
        r.real = off + j;
        const int sp = __ldg(p.sorted_pair + r.real);
        r.w = sp >= 0 ? __ldg(p.topk_w + sp) : 1.0f;
    }
    return r;
}

// One 32 x 32 box of 2-byte values (this lane's row: src, 16 packed pairs) out by a TMA
// store through buffer nb % 2 of the warp's two 2 KB buffers, in the 64-byte swizzle
// (16-byte group j of row r at j ^ ((r / 2) % 4)); a buffer is rewritten once the store
// that used it two boxes ago has read it. nb counts the warp's boxes across units.
MOE_DEV void store_box32(uint8_t* stage, int& nb, const uint32_t (&src)[16], const CUtensorMap* m, int x, int y,
                         int lane) {
    uint8_t* buf = stage + (nb & 1) * 2048;
    if (lane == 0) bulk_wait_read1();
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(src[4 * j], src[4 * j + 1], src[4 * j + 2], src[4 * j + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(m, buf, x, y);
        bulk_commit();
    }
    ++nb;
}

template <int MODE>
MOE_DEV void epilogue(uint32_t tb, const Unit& U, int q, int half, int lane, const Params& p, bool& range_bad,
                      float* stage_out, RowInfo ri, const CUtensorMap* st0, const CUtensorMap* st1, int& nb) {
    const int rit = q * 32 + lane;
    const bool valid = rit < U.rows;
    if (MODE == WG) {
        // each 32 x 32 fp32 block: lane = row into shared memory in the 128-byte swizzle
        // (16-byte group g of row r at g ^ (r % 8): conflict-free), then one TMA store of the
        // box by lane 0 (rows past M are not written); the block's buffer is reused once the
        // previous store has read it
        const CUtensorMap* st = U.e < p.E ? st0 : st1;  // the routed experts' gradient, the shared one's
        const int z = U.e < p.E ? U.e : 0;
#pragma unroll 1
        for (int c = half; c < BN / 32; c += 2) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tb + c * 32, v);
            tmem_ld_wait();
            const int col = U.n * BN + c * 32;
            if (col >= p.N) break;
            if (lane == 0) bulk_wait_read0();
            __syncwarp();
#pragma unroll
            for (int g = 0; g < 8; ++g)
                *reinterpret_cast<uint4*>(stage_out + lane * 32 + ((g ^ (lane & 7)) << 2)) =
                    make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_3d(st, stage_out, col, U.row0 + q * 32, z);
                bulk_commit();
            }
        }
        return;
    }
    // row modes: padded row, its real row (or padding) and the pair's gate weight
    const int64_t prow = int64_t(U.row0) + rit;
    const int real = ri.real;
    const float w = ri.w;
    const int f = p.f, f2 = 2 * p.f;
    const float L = p.limit;
    // padded row counts are multiples of 64, so a warp's 32 rows are all valid or none (the
    // TMA stores of GU and DH write whole 32-row boxes)
    const bool wvalid = q * 32 < U.rows && (U.rows & 31) == 0;
    if (q * 32 < U.rows && (U.rows & 31) != 0 && lane == 0) set_error(p.err, MOE_DEVERR_BOUNDS);
    if (MODE == GU) {
#pragma unroll 1
        for (int c = half; c < 4; c += 2) {
            uint32_t g[32], v[32];
            tmem_ld_32x32b_x32(tb + c * 32, g);
            tmem_ld_32x32b_x32(tb + 128 + c * 32, v);
            tmem_ld_wait();
            const int col = U.n * 128 + c * 32;
            if (wvalid && col < f) {  // warp-uniform: the TMA stores below need every lane
                uint32_t pg[16], pu[16], pw[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
                    const float u0 = __uint_as_float(v[2 * i]), u1 = __uint_as_float(v[2 * i + 1]);
                    const float h0 = tc::swiglu(g0, u0, L), h1 = tc::swiglu(g1, u1, L);
                    const float cg0 = clamp_code(g0, L), cg1 = clamp_code(g1, L);
                    const float cu0 = clamp_code(u0, L), cu1 = clamp_code(u1, L);
                    range_bad |= !(f16_range_ok(h0) && f16_range_ok(h1) && f16_range_ok(cg0) && f16_range_ok(cg1) &&
                                   f16_range_ok(cu0) && f16_range_ok(cu1));
                    pg[i] = pack_f16x2(cg0, cg1);
                    pu[i] = pack_f16x2(cu0, cu1);
                    pw[i] = pack_f16x2(w * h0, w * h1);
                }
                // g, u codes (gu) and w h (hw): three boxes by TMA store (lane 0's row is the
                // warp's first)
                uint8_t* stage = reinterpret_cast<uint8_t*>(stage_out);
                store_box32(stage, nb, pg, st0, col, int(prow), lane);
                store_box32(stage, nb, pu, st0, f + col, int(prow), lane);
                store_box32(stage, nb, pw, st1, col, int(prow), lane);
            }
        }
    } else if (MODE == DH) {
        float dot = 0.f;
        // the chunk's g and u (fp16), 8 vector loads issued together, one chunk ahead: the
        // next chunk's are in flight while this one is computed and stored
        auto load_gu = [&](int c, uint4 (&gq)[4], uint4 (&uq)[4]) {
            const int col = U.n * BN + c * 32;
            if (valid && col < f && c < BN / 32) {
                const uint4* gsrc = reinterpret_cast<const uint4*>(p.gu + prow * f2 + col);
                const uint4* usrc = reinterpret_cast<const uint4*>(p.gu + prow * f2 + f + col);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    gq[i] = gsrc[i];
                    uq[i] = usrc[i];
                }
            }
        };
        uint4 gn[4], un[4];
        load_gu(half, gn, un);
#pragma unroll 1
        for (int c = half; c < BN / 32; c += 2) {
            uint4 gq4[4], uq4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                gq4[i] = gn[i];
                uq4[i] = un[i];
            }
            load_gu(c + 2, gn, un);
            uint32_t v[32];
            tmem_ld_32x32b_x32(tb + c * 32, v);
            tmem_ld_wait();
            const int col = U.n * BN + c * 32;
            if (wvalid && col < f) {  // warp-uniform: the TMA stores below need every lane
                // h = silu(gc) uc is recomputed from g and u for the routing-weight dot
                const uint32_t* gw = reinterpret_cast<const uint32_t*>(gq4);
                const uint32_t* uw = reinterpret_cast<const uint32_t*>(uq4);
                uint32_t pg[16], pu[16], qg[16], qu[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const uint32_t gg = gw[i / 2], uu = uw[i / 2];
                    float dgv[2], duv[2];
#pragma unroll
                    for (int s2 = 0; s2 < 2; ++s2) {
                        const float dhu = __uint_as_float(v[i + s2]);
                        const float gv = s2 ? f16_hi(gg) : f16_lo(gg), uv = s2 ? f16_hi(uu) : f16_lo(uu);
                        const float gc = L > 0.f ? fminf(fmaxf(gv, -L), L) : gv;
                        const float uc = L > 0.f ? fminf(fmaxf(uv, -L), L) : uv;
                        float sg;
                        const float sl = silu_f(gc, sg);
                        dot += sl * uc * dhu;  // h = silu(gc) uc
                        const float dh = w * dhu;
                        const bool pg_ = !(L > 0.f) || fabsf(gv) <= L;
                        const bool pu_ = !(L > 0.f) || fabsf(uv) <= L;
                        dgv[s2] = pg_ ? dh * uc * sg * (1.0f + gc * (1.0f - sg)) : 0.f;
                        duv[s2] = pu_ ? dh * sl : 0.f;
                    }
                    pg[i / 2] = pack_bf16x2(dgv[0], dgv[1]);
                    pu[i / 2] = pack_bf16x2(duv[0], duv[1]);
                    range_bad |= !(f16_range_ok(dgv[0]) && f16_range_ok(dgv[1]) && f16_range_ok(duv[0]) &&
                                   f16_range_ok(duv[1]));
                    qg[i / 2] = pack_f16x2(dgv[0], dgv[1]);
                    qu[i / 2] = pack_f16x2(duv[0], duv[1]);
                }
                // the chunk's four 32 x 32 boxes (dg, du in bf16, then in fp16) leave by TMA
                // stores through this warp's two 2 KB buffers (64-byte swizzle: 16-byte group j
                // of row r at j ^ ((r / 2) % 4)); a buffer is rewritten once the store that
                // used it two boxes ago has read it. The warp's 32 rows are all inside the
                // expert's padded rows (their count is a multiple of 64), so whole boxes go out.
                uint8_t* stage = reinterpret_cast<uint8_t*>(stage_out);
                store_box32(stage, nb, pg, st0, col, int(prow), lane);  // bf16
                store_box32(stage, nb, pu, st0, f + col, int(prow), lane);
                store_box32(stage, nb, qg, st1, col, int(prow), lane);  // fp16
                store_box32(stage, nb, qu, st1, f + col, int(prow), lane);
            }
        }
        if (real >= 0) p.dwp[(int64_t(real) * p.n_tiles + U.n) * 2 + half] = dot;
    } else {  // DX
#pragma unroll 1
        for (int c = half; c < BN / 32; c += 2) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tb + c * 32, v);
            tmem_ld_wait();
            const int col = U.n * BN + c * 32;
            if (real >= 0 && col < p.d) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float a = __uint_as_float(v[2 * i]), b = __uint_as_float(v[2 * i + 1]);
                    range_bad |= !(f16_range_ok(a) && f16_range_ok(b));
                    pk[i] = pack_f16x2(a, b);
                }
                uint4* dst = reinterpret_cast<uint4*>(p.dxr + int64_t(real) * p.d + col);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
        }
    }
}

// Operand maps per mode:
//   GU: A = xg; B0/B1 = W_gate/W_up (N-major, 2 chunks a copy), S0/S1 the shared expert's.
//   DH: A = dout rows; B0 = W_down read K-major ([E, f, d] as N = f rows of K = d); S0 shared.
//   DX: A = [dg|du]; B0/B1 = W_gate/W_up read K-major ([E, d, f] as N = d rows of K = f); S0/S1 shared.
//   WG: A = (w h)^T or xg^T [M, rp]; B0 = the activation rows, N-major (4 chunks a copy).
// TMA store maps O0 / O1: GU g|u and w h (fp16); DH dg|du in bf16 and in fp16; WG the
// routed experts' and the shared expert's gradient (fp32); DX none.
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmS0,
                    const __grid_constant__ CUtensorMap tmS1, const __grid_constant__ CUtensorMap tmO0,
                    const __grid_constant__ CUtensorMap tmO1, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* tfull = empty + kStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint64_t* ufull = drain + 1;
    uint64_t* uempty = ufull + UR;
    volatile int* unit_ring = reinterpret_cast<volatile int*>(uempty + UR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(unit_ring) + UR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* stage_out = reinterpret_cast<float*>(smem + kStages * kStageBytes + 1024);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, kEpiWarps);
        }
        for (int r = 0; r < UR; ++r) {
            mbar_init(ufull + r, 1);
            mbar_init(uempty + r, kUnitReaders);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB0);
        tma_prefetch_desc(&tmB1);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    griddep_wait();
    griddep_launch();

    int total_units;
    if (MODE == WG)
        total_units = __ldg(p.wbase + p.Etot) * ((p.M + BM - 1) / BM) * ((p.N + BN - 1) / BN);
    else
        total_units = __ldg(p.tile_base + p.Etot) * p.n_tiles;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        int stage = 0;
        uint32_t phase = 0, issued = 0, issued_par = 0;
        bool ok = true;
        int uslot = 0;
        uint32_t uphase = 0;
        while (ok) {
            int u = -1;
            if (!tc::ring_publish(u, uslot, uphase, p.unit_counter, total_units, unit_ring, ufull, uempty,
                                  abort_flag, p.err, p.wait_ns)) {
                ok = false;
                break;
            }
            if (u < 0) break;
            const Unit U = decode<MODE>(u, p);
            const bool sh = U.e >= p.E;
            const int z = sh ? 0 : U.e;
            const int kb_half = p.f / BK;  // DX: k-blocks of W_gate, then of W_up
            const int po = MODE == WG ? __ldg(p.poff + U.e) : 0;
            for (int kb = 0; kb < U.kb; ++kb) {
                int okl = 1;
                if (lane == 0) okl = mbar_wait_bounded(empty + stage, phase ^ 1u, abort_flag, p.err, p.wait_ns);
                okl = __shfl_sync(0xFFFFFFFFu, okl, 0);
                if (!okl) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    uint8_t* sa = smem + stage * kStageBytes;
                    uint8_t* sb = sa + A_BYTES;
                    mbar_arrive_expect_tx(full + stage, A_BYTES + B_BYTES);
                    if (MODE == WG) {
                        // A: 128 M-columns of the row buffer (two 64-wide chunks) x 64 K-rows, N-major
                        tma_load_4d(sa, &tmA, full + stage, 0, po + kb * BK, 2 * U.m, 0);
                        tma_load_4d(sb, &tmB0, full + stage, 0, po + kb * BK, 4 * U.n, 0);
                    } else {
                        tma_load_2d(sa, &tmA, full + stage, kb * BK, U.row0);
                        if (MODE == GU) {
                            tma_load_4d(sb, sh ? &tmS0 : &tmB0, full + stage, 0, kb * BK, 2 * U.n, z);
                            tma_load_4d(sb + 2 * B_CHUNK, sh ? &tmS1 : &tmB1, full + stage, 0, kb * BK, 2 * U.n, z);
                        } else if (MODE == DH) {
                            tma_load_3d(sb, sh ? &tmS0 : &tmB0, full + stage, kb * BK, U.n * BN, z);
                        } else {  // DX
                            if (kb < kb_half)
                                tma_load_3d(sb, sh ? &tmS0 : &tmB0, full + stage, kb * BK, U.n * BN, z);
                            else
                                tma_load_3d(sb, sh ? &tmS1 : &tmB1, full + stage, (kb - kb_half) * BK, U.n * BN, z);
                        }
                    }
                    issued |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                }
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
            for (int s = 0; s < kStages; ++s)
                if (issued >> s & 1u) mbar_wait_bounded(full + s, (issued_par >> s) & 1u, nullptr, p.err, kDrainLimitNs);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        constexpr bool kBmn = MODE == GU || MODE == WG;  // B N-major (else K-major)
        constexpr bool kAmn = MODE == WG;                // A N-major (else K-major)
        constexpr int kBf16 = (MODE == GU || MODE == DX) ? 1 : 0;  // else fp16 x fp16
        constexpr uint32_t IDESC = idesc_f16_f32(BM, BN, kBf16, kAmn ? 1 : 0, kBmn ? 1 : 0);
        int stage = 0, acc = 0;
        uint32_t phase = 0, acc_phase = 0;
        bool ok = true;
        int uslot = 0;
        uint32_t uphase = 0;
        while (ok) {
            int u = -1;
            if (!tc::ring_read(u, uslot, uphase, unit_ring, ufull, uempty, abort_flag, p.err, p.wait_ns)) break;
            if (u < 0) break;
            int okl = 1;
            if (lane == 0) okl = mbar_wait_bounded(tempty + acc, acc_phase ^ 1u, abort_flag, p.err, p.wait_ns);
            okl = __shfl_sync(0xFFFFFFFFu, okl, 0);
            if (!okl) break;
            tc_fence_after();
            const int KB = decode<MODE>(u, p).kb;
            const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
            for (int kb = 0; kb < KB; ++kb) {
                if (lane == 0) okl = mbar_wait_bounded(full + stage, phase, abort_flag, p.err, p.wait_ns);
                okl = __shfl_sync(0xFFFFFFFFu, okl, 0);
                if (!okl) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t a0 = smem_u32(smem + stage * kStageBytes);
                    const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
                    for (int jj = 0; jj < BK / 16; ++jj) {
                        const uint64_t ad =
                            kAmn ? sdesc_sw128(a0 + jj * 2048, B_CHUNK, 1024) : sdesc_sw128(a0 + jj * 32, 16, 1024);
                        const uint64_t bd =
                            kBmn ? sdesc_sw128(b0 + jj * 2048, B_CHUNK, 1024) : sdesc_sw128(b0 + jj * 32, 16, 1024);
                        umma_bf16(d_tmem, ad, bd, IDESC, (kb | jj) != 0);
                    }
                    umma_commit(empty + stage);
                }
                __syncwarp();
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) umma_commit(tfull + acc);
            __syncwarp();
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0) {
            umma_commit(drain);
            mbar_wait_bounded(drain, 0, nullptr, p.err, kDrainLimitNs);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 2 .. 2+kEpiWarps-1)
        const int q = warp & 3;                // TMEM lanes 32q .. 32q+31
        const int half = (warp - 2) / 4;       // every other 32-column chunk
        int acc = 0;
        uint32_t acc_phase = 0;
        bool range_bad = false;
        int uslot = 0;
        uint32_t uphase = 0;
        int nb = 0;  // TMA store boxes of this warp (GU, DH)
        while (true) {
            int u = -1;
            if (!tc::ring_read(u, uslot, uphase, unit_ring, ufull, uempty, abort_flag, p.err, p.wait_ns)) break;
            if (u < 0) break;
            const Unit U = decode<MODE>(u, p);
            const RowInfo ri = MODE == WG ? RowInfo{-1, 0.f} : row_info(U, q, lane, p);
            int okl = 1;
            if (lane == 0) okl = mbar_wait_bounded(tfull + acc, acc_phase, abort_flag, p.err, p.wait_ns);
            okl = __shfl_sync(0xFFFFFFFFu, okl, 0);
            if (!okl) break;
            tc_fence_after();
            const uint32_t tb = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * BN);
            epilogue<MODE>(tb, U, q, half, lane, p, range_bad, stage_out + (warp - 2) * 32 * 32, ri, &tmO0, &tmO1,
                           nb);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty + acc);
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (range_bad) set_error(p.err, MOE_DEVERR_RANGE);
        if (MODE != DX && lane == 0) bulk_wait0();  // this warp's TMA stores are complete
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------- small kernels

// One block of 512 threads, thread e owns expert e (Etot <= 257): padded
// offsets, 128-row tile prefix over the padded rows, prefix of experts with
// rows; zeroes the GEMMs' unit counters.
__global__ void __launch_bounds__(512) bwd_schedule_kernel(const int32_t* __restrict__ offsets, int Etot,
                                                           int32_t* __restrict__ poff, int32_t* __restrict__ tile_base,
                                                           int32_t* __restrict__ wbase, int32_t* __restrict__ counters,
                                                           uint32_t* err) {
    __shared__ int sums[3][16];
    griddep_wait();
    griddep_launch();
    const int e = threadIdx.x, lane = e & 31, w = e >> 5;
    int r = 0;
    if (e < Etot) {
        r = offsets[e + 1] - offsets[e];
        if (r < 0) {
            set_error(err, MOE_DEVERR_BOUNDS);
            r = 0;
        }
    }
    const int rp = (r + kPad - 1) / kPad * kPad;
    const int mt = (rp + BM - 1) / BM;
    const int tw = r > 0 ? 1 : 0;
    int a = rp, b = mt, c = tw;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int x = __shfl_up_sync(0xFFFFFFFFu, a, off);
        const int y = __shfl_up_sync(0xFFFFFFFFu, b, off);
        const int z = __shfl_up_sync(0xFFFFFFFFu, c, off);
        if (lane >= off) {
            a += x;
            b += y;
            c += z;
        }
    }
    if (lane == 31) {
        sums[0][w] = a;
        sums[1][w] = b;
        sums[2][w] = c;
    }
    __syncthreads();
    int ba = 0, bb = 0, bc = 0;
    for (int i = 0; i < w; ++i) {
        ba += sums[0][i];
        bb += sums[1][i];
        bc += sums[2][i];
    }
    if (e <= Etot) {  // e == Etot holds the totals (its own terms are zero)
        poff[e] = ba + a - rp;
        tile_base[e] = bb + b - mt;
        wbase[e] = bc + c - tw;
    }
    if (e < 8) counters[e] = 0;
}

// One warp per padded row (grid-stride): xg = x[token] (bf16, for the products
// with the bf16 gate/up weights) and its fp16 copy xg16 (exact for x in fp16's
// range; for the weight gradients), dog = fp16(dout[token]); zero for padding
// rows. Rows past poff[Etot] are not touched.
__global__ void __launch_bounds__(256) bwd_gather_kernel(const uint16_t* __restrict__ x, const float* __restrict__ dout,
                                                         const int32_t* __restrict__ sorted_token,
                                                         const int32_t* __restrict__ offsets,
                                                         const int32_t* __restrict__ poff, int Etot, int T, int d,
                                                         uint16_t* __restrict__ xg, uint16_t* __restrict__ xg16,
                                                         uint16_t* __restrict__ dog, uint32_t* err) {
    griddep_wait();
    griddep_launch();
    const int lane = threadIdx.x & 31;
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
    const int total = poff[Etot];
    bool bad = false;
    for (int64_t pr = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); pr < total; pr += warps) {
        int lo = 0, hi = Etot;  // poff[lo] <= pr < poff[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(poff + mid) <= pr) lo = mid;
            else hi = mid;
        }
        const int j = int(pr) - __ldg(poff + lo);
        const int off = __ldg(offsets + lo);
        int t = -1;
        if (j < __ldg(offsets + lo + 1) - off) {
            t = __ldg(sorted_token + off + j);
            if (t < 0 || t >= T) {
                set_error(err, MOE_DEVERR_BOUNDS);
                t = -1;
            }
        }
        uint4* xo = reinterpret_cast<uint4*>(xg + pr * d);
        uint4* xh = reinterpret_cast<uint4*>(xg16 + pr * d);
        uint4* go = reinterpret_cast<uint4*>(dog + pr * d);
        for (int c = lane; c < d / 8; c += 32) {
            uint4 xv = make_uint4(0, 0, 0, 0), gv = make_uint4(0, 0, 0, 0);
            if (t >= 0) {
                xv = __ldg(reinterpret_cast<const uint4*>(x + int64_t(t) * d) + c);
                const float4* s = reinterpret_cast<const float4*>(dout + int64_t(t) * d) + 2 * c;
                const float4 a = __ldg(s), b = __ldg(s + 1);
                gv = make_uint4(pack_f16x2(a.x, a.y), pack_f16x2(a.z, a.w), pack_f16x2(b.x, b.y),
                                pack_f16x2(b.z, b.w));
                bad |= !(f16_range_ok(a.x) && f16_range_ok(a.y) && f16_range_ok(a.z) && f16_range_ok(a.w) &&
                         f16_range_ok(b.x) && f16_range_ok(b.y) && f16_range_ok(b.z) && f16_range_ok(b.w));
            }
            xo[c] = xv;
            xh[c] = make_uint4(bf16x2_to_f16x2(xv.x), bf16x2_to_f16x2(xv.y), bf16x2_to_f16x2(xv.z),
                               bf16x2_to_f16x2(xv.w));
            go[c] = gv;
        }
    }
    if (bad) set_error(err, MOE_DEVERR_RANGE);
}

// d topk_w[p] = sum over the DH n-tiles (and both epilogue halves, in order) of
// <h, dhu> of the pair's row; 0 if dropped.
__global__ void __launch_bounds__(256) dw_reduce_kernel(const int32_t* __restrict__ pair_row,
                                                        const float* __restrict__ dwp, int64_t pairs, int nt,
                                                        int64_t rows, float* __restrict__ d_topk_w, uint32_t* err) {
    griddep_wait();
    griddep_launch();
    for (int64_t q = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; q < pairs; q += int64_t(gridDim.x) * blockDim.x) {
        int r = pair_row[q];
        if (r >= rows) {
            set_error(err, MOE_DEVERR_BOUNDS);
            r = -1;
        }
        float s = 0.f;
        if (r >= 0)
            for (int n = 0; n < 2 * nt; ++n) s += dwp[int64_t(r) * 2 * nt + n];
        d_topk_w[q] = s;
    }
}

// dlogits: one warp per token; dl_j = w_j (dw_j - sum_i w_i dw_i) on the k
// selected experts, 0 elsewhere ("mini-AGI PR #3" requested(): softmax over the
// selected, renormalised).
__global__ void __launch_bounds__(256) route_backward_kernel(const int32_t* __restrict__ topk_idx,
                                                             const float* __restrict__ topk_w,
                                                             const float* __restrict__ d_topk_w, int T, int E, int k,
                                                             float* __restrict__ dlogits) {
    griddep_wait();
    griddep_launch();
    const int lane = threadIdx.x & 31;
    const int64_t t = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float wj = lane < k ? topk_w[t * k + lane] : 0.f;
    const float dj = lane < k ? d_topk_w[t * k + lane] : 0.f;
    float s = wj * dj;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, off);
    for (int e = lane; e < E; e += 32) dlogits[t * E + e] = 0.f;
    __syncwarp();
    if (lane < k) {
        const int e = topk_idx[t * k + lane];
        if (e >= 0 && e < E) dlogits[t * E + e] = wj * (dj - s);
    }
}

// Weight gradients of routed experts without rows are zero (no GEMM unit writes them).
__global__ void __launch_bounds__(256) zero_untouched_kernel(const int32_t* __restrict__ offsets, int E,
                                                             int64_t per_expert, float* __restrict__ a,
                                                             float* __restrict__ b, float* __restrict__ c) {
    griddep_wait();
    griddep_launch();
    const int e = blockIdx.y;
    if (offsets[e + 1] > offsets[e]) return;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < per_expert; i += int64_t(gridDim.x) * blockDim.x) {
        a[e * per_expert + i] = 0.f;
        b[e * per_expert + i] = 0.f;
        c[e * per_expert + i] = 0.f;
    }
}

template <int MODE>
cudaError_t launch_mode(const CUtensorMap& A, const CUtensorMap& B0, const CUtensorMap& B1, const CUtensorMap& S0,
                        const CUtensorMap& S1, const CUtensorMap& O0, const CUtensorMap& O1, const Params& p,
                        cudaStream_t s) {
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        const cudaError_t e = cudaFuncSetAttribute(bwd_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   kSmem);
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    {
        ProfScope prof_(MOE_K_BWD_GEMM, s);
        const cudaError_t le =
            launch_pdl(false, bwd_gemm_kernel<MODE>, dim3(num_sms()), dim3(kThreads), kSmem, s, A, B0, B1, S0, S1, O0,
                       O1, p);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace bwd

namespace tc {
bool map_weights_kmajor(CUtensorMap* m, const void* base, int nexp, int N, int K, bool f16 = false);
bool map_f32_tiles(CUtensorMap* m, const void* base, int nexp, int M, int N);
bool map_rows_store32(CUtensorMap* m, const void* base, int64_t rows, int cols, bool f16);
bool map_act_mn(CUtensorMap* m, const void* base, int64_t rows, int N, int64_t row_stride, int chunks);
}  // namespace tc

int64_t bwd_padded_rows(const Dims& D) { return (D.rows + bwd::kPad - 1) / bwd::kPad * bwd::kPad + int64_t(bwd::kPad) * D.Etot; }

cudaError_t launch_backward(const Dims& D, const BwdArgs& a, cudaStream_t s) {
    using namespace bwd;
    const int64_t rp = bwd_padded_rows(D);
    const int Etot = D.Etot, d = D.d, f = D.f;
    uint8_t* ws = a.ws;
    const WsLayout& L = a.layout;
    int32_t* poff = reinterpret_cast<int32_t*>(ws + L.b_poff);
    int32_t* tile_base = reinterpret_cast<int32_t*>(ws + L.b_tile_base);
    int32_t* wbase = reinterpret_cast<int32_t*>(ws + L.b_wbase);
    int32_t* counters = reinterpret_cast<int32_t*>(ws + L.b_counters);
    uint16_t* xg = reinterpret_cast<uint16_t*>(ws + L.b_xg);
    uint16_t* xg16 = reinterpret_cast<uint16_t*>(ws + L.b_xg16);
    uint16_t* dog = reinterpret_cast<uint16_t*>(ws + L.b_dog);
    uint16_t* gu = reinterpret_cast<uint16_t*>(ws + L.b_gu);
    uint16_t* hw = reinterpret_cast<uint16_t*>(ws + L.b_hw);
    uint16_t* dgu = reinterpret_cast<uint16_t*>(ws + L.b_dgu);
    uint16_t* dgu16 = reinterpret_cast<uint16_t*>(ws + L.b_dgu16);
    uint16_t* dxr = reinterpret_cast<uint16_t*>(ws + L.b_dxr);
    float* dwp = reinterpret_cast<float*>(ws + L.b_dwp);
    cudaError_t e;
    {
        ProfScope prof_(MOE_K_BWD_SMALL, s);
        if ((e = launch_pdl(false, bwd_schedule_kernel, dim3(1), dim3(512), 0, s, a.offsets, Etot, poff, tile_base,
                            wbase, counters, a.err)) != cudaSuccess)
            return e;
    }
    {
        ProfScope prof_(MOE_K_BWD_SMALL, s);
        int64_t blocks = (rp + 7) / 8;
        if (blocks > int64_t(num_sms()) * 8) blocks = int64_t(num_sms()) * 8;
        if ((e = launch_pdl(false, bwd_gather_kernel, dim3(int(blocks)), dim3(256), 0, s, a.x, a.dout, a.sorted_token,
                            a.offsets, poff, Etot, D.T, d, xg, xg16, dog, a.err)) != cudaSuccess)
            return e;
    }
    const moe_weights* w = a.w;
    CUtensorMap mX, mDog, mDgu, mHwN, mXgN;
    CUtensorMap mG, mU, mGk, mUk, mDk, sG, sU, sGk, sUk, sDk, mDogN, mDgN, mDuN;
    if (!tc::map_rows(&mX, xg, rp, d) || !tc::map_rows(&mDog, dog, rp, d) || !tc::map_rows(&mDgu, dgu, rp, 2 * f) ||
        !tc::map_act_mn(&mHwN, hw, rp, f, f, 2) || !tc::map_act_mn(&mXgN, xg16, rp, d, d, 2) ||
        !tc::map_weights(&mG, w->w_gate, D.E, d, f, 2) || !tc::map_weights(&mU, w->w_up, D.E, d, f, 2) ||
        !tc::map_weights_kmajor(&mGk, w->w_gate, D.E, d, f) || !tc::map_weights_kmajor(&mUk, w->w_up, D.E, d, f) ||
        !tc::map_weights_kmajor(&mDk, w->w_down, D.E, f, d, true) || !tc::map_act_mn(&mDogN, dog, rp, d, d, 4) ||
        !tc::map_act_mn(&mDgN, dgu16, rp, f, 2 * int64_t(f), 4) ||
        !tc::map_act_mn(&mDuN, dgu16 + f, rp, f, 2 * int64_t(f), 4))
        return cudaErrorInvalidValue;
    if (D.has_shared) {
        if (!tc::map_weights(&sG, w->shared_gate, 1, d, f, 2) || !tc::map_weights(&sU, w->shared_up, 1, d, f, 2) ||
            !tc::map_weights_kmajor(&sGk, w->shared_gate, 1, d, f) ||
            !tc::map_weights_kmajor(&sUk, w->shared_up, 1, d, f) ||
            !tc::map_weights_kmajor(&sDk, w->shared_down, 1, f, d, true))
            return cudaErrorInvalidValue;
    } else {
        sG = mG;
        sU = mU;
        sGk = mGk;
        sUk = mUk;
        sDk = mDk;
    }
    Params p{};
    p.E = D.E;
    p.Etot = Etot;
    p.d = d;
    p.f = f;
    p.rp = rp;
    p.tile_base = tile_base;
    p.poff = poff;
    p.wbase = wbase;
    p.offsets = a.offsets;
    p.sorted_pair = a.sorted_pair;
    p.topk_w = a.topk_w;
    p.limit = D.limit;
    p.gu = gu;
    p.hw = hw;
    p.dgu = dgu;
    p.dgu16 = dgu16;
    p.dxr = dxr;
    p.dwp = dwp;
    p.err = a.err;
    p.wait_ns = a.wait_ns;
    const int nt_dh = (f + BN - 1) / BN;
    // GU: g, u, h, (w h)^T
    p.K = d;
    p.n_tiles = (f + 127) / 128;
    p.unit_counter = counters + 0;
    {
        // GU's TMA store maps: the g|u codes and w h (fp16)
        CUtensorMap stGU, stHW;
        if (!tc::map_rows_store32(&stGU, gu, rp, 2 * f, true) || !tc::map_rows_store32(&stHW, hw, rp, f, true))
            return cudaErrorInvalidValue;
        if ((e = launch_mode<GU>(mX, mG, mU, sG, sU, stGU, stHW, p, s)) != cudaSuccess) return e;
    }
    // DH: dg, du; <h, dhu> partials
    p.K = d;
    p.n_tiles = nt_dh;
    p.unit_counter = counters + 1;
    {
        // DH's TMA store maps: dg|du in bf16 and in fp16
        CUtensorMap stB, stH;
        if (!tc::map_rows_store32(&stB, dgu, rp, 2 * f, false) || !tc::map_rows_store32(&stH, dgu16, rp, 2 * f, true))
            return cudaErrorInvalidValue;
        if ((e = launch_mode<DH>(mDog, mDk, mDk, sDk, sDk, stB, stH, p, s)) != cudaSuccess) return e;
    }
    // DX: dx rows
    p.K = 2 * f;
    p.n_tiles = (d + BN - 1) / BN;
    p.unit_counter = counters + 2;
    if ((e = launch_mode<DX>(mDgu, mGk, mUk, sGk, sUk, mDgu, mDgu, p, s)) != cudaSuccess) return e;
    // WG: dW_down = (w h)^T dout_rows [f, d]; dW_gate = xg^T dg, dW_up = xg^T du [d, f]; its
    // TMA store maps: the routed experts' gradient and the shared expert's (the routed map
    // again without one).
    auto wg = [&](const CUtensorMap& A, const CUtensorMap& B, float* dw, float* sdw, int M, int N,
                  int32_t* counter) -> cudaError_t {
        CUtensorMap stD, stS;
        if (!tc::map_f32_tiles(&stD, dw, D.E, M, N) || (sdw && !tc::map_f32_tiles(&stS, sdw, 1, M, N)))
            return cudaErrorInvalidValue;
        if (!sdw) stS = stD;
        p.M = M;
        p.N = N;
        p.dw = dw;
        p.sdw = sdw;
        p.unit_counter = counter;
        return launch_mode<WG>(A, B, B, B, B, stD, stS, p, s);
    };
    float* sd = D.has_shared ? a.g->dshared_down : nullptr;
    float* sg = D.has_shared ? a.g->dshared_gate : nullptr;
    float* su = D.has_shared ? a.g->dshared_up : nullptr;
    if ((e = wg(mHwN, mDogN, a.g->dw_down, sd, f, d, counters + 3)) != cudaSuccess) return e;
    if ((e = wg(mXgN, mDgN, a.g->dw_gate, sg, d, f, counters + 4)) != cudaSuccess) return e;
    if ((e = wg(mXgN, mDuN, a.g->dw_up, su, d, f, counters + 5)) != cudaSuccess) return e;
    {
        ProfScope prof_(MOE_K_BWD_SMALL, s);
        const int64_t per = int64_t(d) * f;
        if ((e = launch_pdl(false, zero_untouched_kernel, dim3(64, D.E), dim3(256), 0, s, a.offsets, D.E, per,
                            a.g->dw_gate, a.g->dw_up, a.g->dw_down)) != cudaSuccess)
            return e;
    }
    // dx = sum of each token's dx rows (+ the shared expert's)
    Dims Dc = D;
    Dc.out_bf16 = 0;
    if ((e = launch_combine(Dc, dxr, a.pair_row, a.offsets, a.g->dx, s)) != cudaSuccess) return e;
    {
        ProfScope prof_(MOE_K_BWD_SMALL, s);
        int64_t blocks = (D.pairs + 255) / 256;
        if (blocks > int64_t(num_sms()) * 8) blocks = int64_t(num_sms()) * 8;
        if (blocks < 1) blocks = 1;
        if ((e = launch_pdl(false, dw_reduce_kernel, dim3(int(blocks)), dim3(256), 0, s, a.pair_row, dwp, D.pairs,
                            nt_dh, int64_t(D.rows), a.g->d_topk_w, a.err)) != cudaSuccess)
            return e;
    }
    if (a.g->dlogits && a.topk_idx) {
        ProfScope prof_(MOE_K_BWD_SMALL, s);
        if ((e = launch_pdl(false, route_backward_kernel, dim3((D.T + 7) / 8), dim3(256), 0, s, a.topk_idx, a.topk_w,
                            a.g->d_topk_w, D.T, D.E, D.k, a.g->dlogits)) != cudaSuccess)
            return e;
    }
    return cudaGetLastError();
}

}  // namespace moe

// stream.cu — S8: the few-rows variant for experts with a handful of rows
// (decode). It streams each touched expert's weights once at HBM rate and
// never reads an expert that got no rows.
//
// Prior art: "mini-AGI PR #3" run() subset dispatch — a character being
// written reaches top_k experts, and reading every expert's weights made
// decode bound by memory bandwidth; only the chosen experts are read.
// "Strata PR #4366" — the light kernels own experts with at most 16 rows;
// "TensorFold PR #1607" — K-parallel tiles for plans with few pairs per item.
//
// Work item = (expert, output columns, K slice, chunk of <= 8 rows): 64
// columns of W_gate and of W_up, or 256 columns of W_down. One CTA per SM,
// persistent, everything through one TMA ring (204 KB gate/up, 198 KB down):
//   warp 0     TMA producer: per 64-K block, the 64 x 64 weight boxes (gate
//              and up, or four of down; 128-byte swizzle) and the 8 x 64 tile
//              of the chunk's rows (gathered x, or h; 128-byte swizzle).
//   warps 1-4  consumers, 16 columns of gate and up each, or 64 columns of
//              down: ldmatrix.trans turns the stored [k][n] weight box into the
//              A operand (16 n x 16 k) of mma.sync m16n8k16; the rows tile
//              gives the N=8 operand. fp32 accumulate. The tensor pipe only
//              keeps the instruction count per weight byte low so the kernel
//              stays HBM-bound.
// Gate/up (bf16 x and weights) with one K slice applies the clamped SwiGLU and
// writes h (fp16); with several, fp32 partials go to the workspace and
// stream_reduce finishes (fixed order, deterministic). Down runs in fp16 (h is
// fp16; W_down prepared as fp16, or converted in registers after ldmatrix) and
// writes y = w_pair * (h W_down) (fp16). All waits are bounded; no TMA
// copy into another CTA; no named barriers, so an abort never strands a warp.
#include "internal.h"

namespace moe {

namespace st {

constexpr int NS = 64;               // columns of one weight box (128 bytes of a row)
constexpr int BKS = 64;              // K-rows per stage
constexpr int TILE = BKS * NS * 2;   // weight box, 8 KB
constexpr int XT = 8 * BKS * 2;      // rows tile (8 rows x 64 K), 1 KB
constexpr int CONSUMERS = 4;
constexpr int THREADS = 32 * (CONSUMERS + 1);
constexpr int RC = 8;                // rows per chunk (mma N)

// Per matrix: gate/up items are 64 columns of W_gate and of W_up (two boxes a
// stage, 16 columns of each per consumer warp); down items are 256 columns of
// W_down (four boxes a stage, 64 columns per warp), so each weight row is read
// as 512 contiguous bytes — 64-column down items left HBM half idle.
// FOLD (down only): the gate/up ran K-split and its fp32 partials are summed
// here, into an [RC rows, f] fp16 buffer of h per chunk (no reduce kernel, no
// rows tile in the stages).
template <int MODE, bool FOLD = false>
struct SCfg {
    static constexpr int NMAT = MODE == 0 ? 2 : 4;                // weight boxes per stage
    static constexpr int NSU = MODE == 0 ? NS : 4 * NS;           // output columns per item
    static constexpr int STAGE = NMAT * TILE + (FOLD ? 0 : XT);   // 17 KB / 33 KB (32 KB folded), 1 KB aligned
    static constexpr int STAGES = MODE == 0 ? 12 : 6;
    static constexpr int RING = STAGES * STAGE;                   // 204 KB / 198 KB
    static constexpr int SMEM = 1024 + RING + 512;                // + barriers, abort flag
};
// Row stride of the folded h buffer: 16 bytes past the row, so that the 8 rows a
// consumer warp reads at one k fall in distinct banks.
__host__ __device__ inline int fold_row_bytes(int f) { return 2 * f + 16; }
constexpr int kFoldMaxSmem = 232448;  // dynamic shared memory a block may opt into
inline bool fold_fits(int f) { return SCfg<1, true>::SMEM + RC * fold_row_bytes(f) <= kFoldMaxSmem; }
constexpr int kFoldMaxSlices = 4;  // K-split counts the fold takes (its loads are held in registers)
constexpr int kFoldQ = 3;          // column pairs a consumer thread sums at a time
static_assert((2 * SCfg<0>::STAGES + 3) * 8 <= 512 && (2 * SCfg<1>::STAGES + 3) * 8 <= 512,
              "stage barriers, abort flag and the fold's barriers fit the reserved bytes");

struct StreamParams {
    int mode;            // 0: gate/up, 1: down
    int K, N;            // full reduction length and output width of the matrix
    int kslice, ks;      // K per item and number of K slices
    int E, etot;          // routed experts; with the shared one
    const int32_t* offsets;
    const int32_t* stream_list;
    const int32_t* n_stream;
    const int32_t* sorted_pair;
    const float* topk_w;
    uint16_t* out;        // mode 0: h [rows, f]; mode 1: y_rows [rows, d]
    const float* hpart;   // mode 1 folded: the gate/up partials [ksg, 2, rows, f]
    int ksg;              // mode 1 folded: their K-split count
    float* part;          // mode 0 with ks > 1: [ks, 2, rows, f] fp32
    int64_t rows;
    float limit;
    int down_f16;         // mode 1: W_down already fp16 (no conversion)
    uint32_t* err;
    uint64_t wait_ns;
    // mode 1, every expert streaming (moe_forward of a few tokens): the combine fused in.
    // comb_count: [ceil(N/256)] arrivals per column block, zeroed by the front kernel.
    int32_t* comb_count;
    const int32_t* pair_row;  // [T*k] row of each pair, -1 dropped
    void* comb_out;           // [T, N] fp32, or bf16 with comb_bf16
    int comb_bf16, T, k, has_shared;
};

// The combine of output columns [n0, n0 + 256) for every token, by one warp (8
// columns a lane): the kept pairs' y rows in the fixed order j = 0..k-1, then the
// shared expert's row, summed in fp32 as combine_kernel does. y rows are read
// from L2 (other SMs wrote them).
MOE_DEV void combine_columns(const StreamParams& p, int n0, int lane) {
    const int c = n0 + lane * 8;
    if (c >= p.N) return;
    const int shared_base = p.has_shared ? __ldg(p.offsets + p.E) : 0;
    for (int t = 0; t < p.T; ++t) {
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        auto add = [&](const uint4& v) {
            acc[0] += f16_lo(v.x); acc[1] += f16_hi(v.x);
            acc[2] += f16_lo(v.y); acc[3] += f16_hi(v.y);
            acc[4] += f16_lo(v.z); acc[5] += f16_hi(v.z);
            acc[6] += f16_lo(v.w); acc[7] += f16_hi(v.w);
        };
        int rr[kMaxK];
        uint4 yv[kMaxK];
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) rr[j] = j < p.k ? __ldg(p.pair_row + int64_t(t) * p.k + j) : -1;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (rr[j] >= 0) yv[j] = __ldcg(reinterpret_cast<const uint4*>(p.out + int64_t(rr[j]) * p.N + c));
        uint4 ys = make_uint4(0, 0, 0, 0);
        if (p.has_shared) ys = __ldcg(reinterpret_cast<const uint4*>(p.out + int64_t(shared_base + t) * p.N + c));
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (rr[j] >= 0) add(yv[j]);
        if (p.has_shared) add(ys);
        if (p.comb_bf16) {
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]);
            o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]);
            o.w = pack_bf16x2(acc[6], acc[7]);
            *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.comb_out) + int64_t(t) * p.N + c) = o;
        } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.comb_out) + int64_t(t) * p.N + c);
            dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
    }
}

struct SUnit {
    int e, n0, k0, ks, row0, nrows;
};

MOE_DEV SUnit decode(int u, const StreamParams& p, int nsu) {
    const int nsl = (p.N + nsu - 1) / nsu;
    const int per = nsl * p.ks;
    const int i = u / per;
    const int rem = u - i * per;
    SUnit U;
    U.e = __ldg(p.stream_list + i);
    if (U.e < 0 || U.e >= p.etot) {  // never for a list the schedule wrote
        set_error(p.err, MOE_DEVERR_BOUNDS);
        U.e = 0;
    }
    U.n0 = (rem / p.ks) * nsu;
    U.ks = rem % p.ks;
    U.k0 = U.ks * p.kslice;
    U.row0 = __ldg(p.offsets + U.e);
    U.nrows = __ldg(p.offsets + U.e + 1) - U.row0;
    return U;
}

MOE_DEV float swiglu(float g, float u, float L) {
    if (L > 0.f) {
        g = fminf(fmaxf(g, -L), L);
        u = fminf(fmaxf(u, -L), L);
    }
    return __fdividef(g, 1.0f + __expf(-g)) * u;  // as in the tile kernels
}

MOE_DEV void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

MOE_DEV void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                            uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

MOE_DEV void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                           uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

MOE_DEV uint16_t to_f16(float v) { return uint16_t(pack_f16x2(v, 0.f) & 0xFFFFu); }

// MODE 0: two weight tiles (gate, up) per stage; MODE 1: one (down). Plus the rows tile.
template <int MODE, bool FOLD = false>
__global__ void __launch_bounds__(THREADS, 1)
    stream_kernel(const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmW1,
                  const __grid_constant__ CUtensorMap tmS0, const __grid_constant__ CUtensorMap tmS1,
                  const __grid_constant__ CUtensorMap tmX, const StreamParams p) {
    using SC = SCfg<MODE, FOLD>;
    static_assert(!FOLD || MODE == 1, "the fold is the down kernel's");
    constexpr int NMAT = SC::NMAT, NSU = SC::NSU, STAGE = SC::STAGE, STAGES = SC::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + SC::RING);
    uint64_t* empty = full + STAGES;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + STAGES);
    // FOLD: h of the current chunk written (every consumer thread) / read (every consumer thread)
    uint64_t* hready = empty + STAGES + 1;
    uint64_t* hfree = hready + 1;
    uint8_t* hbuf = smem + SC::RING + 512;  // FOLD: [RC][fold_row_bytes(f)] fp16

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, CONSUMERS);
        }
        mbar_init(hready, 32 * CONSUMERS);
        mbar_init(hfree, 32 * CONSUMERS);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // the prologue above touched no global memory; wait for the predecessor here
    // (letting the folded down kernel's producer stream its first weight stages before
    // the wait, as the weights and the item list allow, measured 76.3 -> 76.0 us on
    // single-token decode: its blocks only become resident as the gate/up blocks exit)
    griddep_wait();
    griddep_launch();

    const int total = __ldg(p.n_stream) * ((p.N + NSU - 1) / NSU) * p.ks;
    const int KB = p.kslice / BKS;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        int stage = 0;
        uint32_t phase = 0, issued = 0, issued_par = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < total; u += gridDim.x) {
            const SUnit U = decode(u, p, NSU);
            const bool sh = U.e >= p.E;
            const int wrow = (sh ? 0 : U.e * p.K) + U.k0;  // weight row of k0 in the stacked [E*K, N] view
            const int nchunks = (U.nrows + RC - 1) / RC;
            for (int c = 0; ok && c < nchunks; ++c) {
                for (int kb = 0; kb < KB; ++kb) {
                    int okl = 1;
                    if (lane == 0) okl = mbar_wait_bounded(empty + stage, phase ^ 1u, abort_flag, p.err, p.wait_ns);
                    okl = __shfl_sync(0xFFFFFFFFu, okl, 0);
                    if (!okl) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        uint8_t* dst = smem + stage * STAGE;
                        mbar_arrive_expect_tx(full + stage, STAGE);
                        if (MODE == 0) {
                            tma_load_2d(dst, sh ? &tmS0 : &tmW0, full + stage, U.n0, wrow + kb * BKS);
                            tma_load_2d(dst + TILE, sh ? &tmS1 : &tmW1, full + stage, U.n0, wrow + kb * BKS);
                        } else {
                            // the four boxes in one copy (boxes past N are filled with zeros)
                            tma_load_3d(dst, sh ? &tmS0 : &tmW0, full + stage, 0, wrow + kb * BKS, U.n0 / NS);
                        }
                        if (!FOLD)
                            tma_load_2d(dst + NMAT * TILE, &tmX, full + stage, U.k0 + kb * BKS, U.row0 + c * RC);
                        issued |= 1u << stage;
                        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        // On abort, let every copy already issued land before the CTA can exit.
        if (!ok && lane == 0) {
            for (int s = 0; s < STAGES; ++s)
                if (issued >> s & 1u) mbar_wait_bounded(full + s, (issued_par >> s) & 1u, nullptr, p.err, kDrainLimitNs);
        }
        __syncwarp();
        return;
    }

    // ---------------------------------------------------- consumers (warps 1..4)
    // gate/up: warp cw takes columns cw*16 .. +15 of both boxes (gate, up);
    // down: warp cw takes box cw, i.e. columns cw*64 .. +63, as four 16-column groups.
    constexpr int NG = MODE == 0 ? 1 : 4;  // 16-column groups per warp
    const int cw = warp - 1;
    const int gid = lane >> 2, tig = lane & 3;
    int stage = 0;
    uint32_t phase = 0, hph = 0;
    bool ok = true, range_bad = false;
    const int HS = FOLD ? fold_row_bytes(p.K) : 0;
    for (int u = blockIdx.x; ok && u < total; u += gridDim.x) {
        const SUnit U = decode(u, p, NSU);
        const int nchunks = (U.nrows + RC - 1) / RC;
        for (int c = 0; ok && c < nchunks; ++c) {
            const int rc = min(RC, U.nrows - c * RC);
            float acc0[NG][4], acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int g = 0; g < NG; ++g)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc0[g][i] = 0.f;
            if (FOLD) {
                // h of the chunk's rows from the gate/up partials, slices summed in order (as
                // stream_reduce_kernel does), once every consumer is done with the previous
                // chunk's; the weight stages keep streaming in meanwhile
                int okl = mbar_wait_bounded(hfree, hph ^ 1u, abort_flag, p.err, p.wait_ns);
                if (!__all_sync(0xFFFFFFFFu, okl)) {
                    ok = false;
                    break;
                }
                const int64_t slice = int64_t(p.rows) * p.K;  // g of slice s at 2s, u at 2s + 1
                for (int r = 0; r < rc; ++r) {
                    const float* hrow = p.hpart + (int64_t(U.row0) + c * RC + r) * p.K;
                    // kFoldQ column pairs a thread at a time, every slice's loads issued together
                    for (int q0 = cw * 32 + lane; q0 < p.K / 2; q0 += kFoldQ * 32 * CONSUMERS) {
                        float2 gs[kFoldQ][kFoldMaxSlices], us[kFoldQ][kFoldMaxSlices];
#pragma unroll
                        for (int j = 0; j < kFoldQ; ++j) {
                            const int q = q0 + j * 32 * CONSUMERS;
#pragma unroll
                            for (int sl = 0; sl < kFoldMaxSlices; ++sl)
                                if (sl < p.ksg && q < p.K / 2) {
                                    gs[j][sl] = __ldg(reinterpret_cast<const float2*>(hrow + 2 * sl * slice) + q);
                                    us[j][sl] = __ldg(reinterpret_cast<const float2*>(hrow + (2 * sl + 1) * slice) + q);
                                }
                        }
#pragma unroll
                        for (int j = 0; j < kFoldQ; ++j) {
                            const int q = q0 + j * 32 * CONSUMERS;
                            if (q >= p.K / 2) break;
                            float g0 = 0.f, g1 = 0.f, u0 = 0.f, u1 = 0.f;
#pragma unroll
                            for (int sl = 0; sl < kFoldMaxSlices; ++sl)
                                if (sl < p.ksg) {
                                    g0 += gs[j][sl].x;
                                    g1 += gs[j][sl].y;
                                    u0 += us[j][sl].x;
                                    u1 += us[j][sl].y;
                                }
                            const float h0 = swiglu(g0, u0, p.limit), h1 = swiglu(g1, u1, p.limit);
                            range_bad |= !(f16_range_ok(h0) && f16_range_ok(h1));
                            *reinterpret_cast<uint32_t*>(hbuf + r * HS + 4 * q) = pack_f16x2(h0, h1);
                        }
                    }
                }
                mbar_arrive(hready);
                okl = mbar_wait_bounded(hready, hph, abort_flag, p.err, p.wait_ns);
                if (!__all_sync(0xFFFFFFFFu, okl)) {
                    ok = false;
                    break;
                }
            }
            for (int kb = 0; kb < KB; ++kb) {
                int okl = 1;
                if (lane == 0) okl = mbar_wait_bounded(full + stage, phase, abort_flag, p.err, p.wait_ns);
                okl = __shfl_sync(0xFFFFFFFFu, okl, 0);
                if (!okl) {
                    ok = false;
                    break;
                }
                const uint32_t base0 = smem_u32(smem + stage * STAGE) + (MODE == 0 ? 0 : cw * TILE);
                const uint8_t* xt = smem + stage * STAGE + NMAT * TILE;  // rows tile: row r, k at swizzled spot
#pragma unroll
                for (int k16 = 0; k16 < BKS / 16; ++k16) {
                    // weight box: lane l addresses row (l%8) of 8x8 matrix (l/8): k = k16*16 + 8*(l/16) + l%8,
                    // 16-byte chunk 2*grp + (l/8)%2 of the 128-byte row, stored at chunk ^ (k % 8) (128-byte
                    // swizzle); grp = cw (gate/up) or the 16-column group g (down)
                    const int kr = k16 * 16 + ((lane >> 4) << 3) + (lane & 7);
                    // rows tile: row gid, k = k16*16 + 2*tig (+8): chunk (k/8) ^ gid
                    // (FOLD: row gid of the chunk's h buffer, k from the item's start)
                    const int kx = k16 * 16 + 2 * tig;
                    uint32_t b0, b1;
                    if (FOLD) {
                        const uint8_t* hb = hbuf + gid * HS + (kb * BKS + kx) * 2;
                        b0 = *reinterpret_cast<const uint32_t*>(hb);
                        b1 = *reinterpret_cast<const uint32_t*>(hb + 16);
                    } else {
                        b0 = *reinterpret_cast<const uint32_t*>(xt + gid * 128 + (((kx >> 3) ^ gid) << 4) +
                                                                 (kx & 7) * 2);
                        b1 = *reinterpret_cast<const uint32_t*>(xt + gid * 128 + ((((kx + 8) >> 3) ^ gid) << 4) +
                                                                 ((kx + 8) & 7) * 2);
                    }
#pragma unroll
                    for (int g = 0; g < NG; ++g) {
                        const int grp = MODE == 0 ? cw : g;
                        const int ch = (2 * grp + ((lane >> 3) & 1)) ^ (kr & 7);
                        const uint32_t off = uint32_t(kr * 128 + ch * 16);
                        uint32_t a0, a1, a2, a3;
                        ldmatrix_x4_trans(base0 + off, a0, a1, a2, a3);
                        if (MODE == 0) {
                            // x (bf16) against W_gate / W_up (bf16)
                            mma_bf16_16816(acc0[g], a0, a1, a2, a3, b0, b1);
                            ldmatrix_x4_trans(base0 + TILE + off, a0, a1, a2, a3);
                            mma_bf16_16816(acc1, a0, a1, a2, a3, b0, b1);
                        } else if (p.down_f16) {
                            // h (fp16) against W_down prepared as fp16
                            mma_f16_16816(acc0[g], a0, a1, a2, a3, b0, b1);
                        } else {
                            // h (fp16) against W_down converted bf16 -> fp16 in registers
                            mma_f16_16816(acc0[g], bf16x2_to_f16x2(a0), bf16x2_to_f16x2(a1), bf16x2_to_f16x2(a2),
                                          bf16x2_to_f16x2(a3), b0, b1);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty + stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (FOLD) {
                mbar_arrive(hfree);  // this thread's reads of the chunk's h are done
                hph ^= 1u;
            }
            // acc[g][i]: column n = (cw*16 | cw*64 + 16g) + gid + 8*(i/2), row r = 2*tig + (i%2)
#pragma unroll
            for (int g = 0; g < NG; ++g) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = 2 * tig + (i & 1);
                    const int n = U.n0 + (MODE == 0 ? cw * 16 : cw * 64 + g * 16) + gid + 8 * (i >> 1);
                    if (r >= rc || n >= p.N) continue;
                    const int64_t row = int64_t(U.row0) + c * RC + r;
                    if (MODE == 0) {
                        if (p.ks == 1) {
                            const float h = swiglu(acc0[g][i], acc1[i], p.limit);
                            range_bad |= !f16_range_ok(h);
                            p.out[row * p.N + n] = to_f16(h);
                        } else {
                            p.part[((int64_t(U.ks) * 2 + 0) * p.rows + row) * p.N + n] = acc0[g][i];
                            p.part[((int64_t(U.ks) * 2 + 1) * p.rows + row) * p.N + n] = acc1[i];
                        }
                    } else {
                        const int sp = __ldg(p.sorted_pair + row);
                        const float w = sp >= 0 ? __ldg(p.topk_w + sp) : 1.0f;
                        const float y = w * acc0[g][i];
                        range_bad |= !f16_range_ok(y);
                        p.out[row * p.N + n] = to_f16(y);
                    }
                }
            }
        }
        // Fused combine: once its y stores for the item are made, each consumer warp
        // arrives on the item's column block (fence, then a counter); the warp making the
        // block's last arrival (every streaming expert's item, every consumer warp) sums
        // the block's columns of every token. Which warp that is does not change the sum.
        if (MODE == 1 && p.comb_count && ok) {
            __threadfence();
            __syncwarp();
            int last = 0;
            if (lane == 0)
                last = atomicAdd(p.comb_count + U.n0 / NSU, 1) == __ldg(p.n_stream) * CONSUMERS - 1 ? 1 : 0;
            last = __shfl_sync(0xFFFFFFFFu, last, 0);
            if (last) {
                __threadfence();
                combine_columns(p, U.n0, lane);
            }
        }
    }
    if (range_bad) set_error(p.err, MOE_DEVERR_RANGE);
}

// h = swiglu(sum_ks part_g, sum_ks part_u) for the streaming experts' rows (ks > 1).
// Work item = (streaming expert, 256 columns); each thread owns one column of
// the expert's rows, so its 2*ks loads are independent and in flight together
// (single-token decode: one row per expert, 9 experts x 6 items). The partials
// are summed in slice order, so the result does not depend on the mapping.
__global__ void __launch_bounds__(256) stream_reduce_kernel(const float* __restrict__ part, int ks, int64_t rows,
                                                            int f, const int32_t* __restrict__ offsets,
                                                            const int32_t* __restrict__ stream_list,
                                                            const int32_t* __restrict__ n_stream, float limit,
                                                            uint16_t* __restrict__ h, uint32_t* err) {
    griddep_wait();
    griddep_launch();
    const int n = __ldg(n_stream);
    const int cpe = (f + 255) / 256;  // 256-column items per expert
    bool range_bad = false;
    for (int w = blockIdx.x; w < n * cpe; w += gridDim.x) {
        const int i = w / cpe;
        const int col = (w - i * cpe) * 256 + int(threadIdx.x);
        if (col >= f) continue;
        const int e = __ldg(stream_list + i);
        const int r0 = __ldg(offsets + e), nr = __ldg(offsets + e + 1) - r0;
        for (int r = 0; r < nr; ++r) {
            const int64_t row = int64_t(r0) + r;
            float g = 0.f, u = 0.f;
            for (int s = 0; s < ks; ++s) {
                g += part[((int64_t(s) * 2 + 0) * rows + row) * f + col];
                u += part[((int64_t(s) * 2 + 1) * rows + row) * f + col];
            }
            const float hv = swiglu(g, u, limit);
            range_bad |= !f16_range_ok(hv);
            h[row * f + col] = to_f16(hv);
        }
    }
    if (range_bad) set_error(err, MOE_DEVERR_RANGE);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D map over a row-major [nrows, ncols] 2-byte matrix; box 64 (cols) x box_rows; 128-byte swizzle.
static bool map_2d(CUtensorMap* m, const void* base, int64_t nrows, int ncols, int box_rows) {
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t gd[2] = {cuuint64_t(ncols), cuuint64_t(nrows)};
    cuuint64_t gs[1] = {cuuint64_t(ncols) * 2};
    cuuint32_t bx[2] = {64, cuuint32_t(box_rows)}, es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gd, gs, bx, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same matrix seen as [ncols/64 chunks, nrows, 64] (3-D, 128-byte swizzle):
// one copy brings `chunks` 64 x 64 boxes of adjacent columns, 8 KB apart.
static bool map_chunks(CUtensorMap* m, const void* base, int64_t nrows, int ncols, int chunks) {
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t gd[3] = {64, cuuint64_t(nrows), cuuint64_t(ncols / 64)};
    cuuint64_t gs[2] = {cuuint64_t(ncols) * 2, 128};
    cuuint32_t bx[3] = {64, BKS, cuuint32_t(chunks)}, es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gd, gs, bx, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// smem: the dynamic shared memory of this launch (SCfg::SMEM, plus the h buffer when folded).
template <int MODE, bool FOLD = false>
static cudaError_t launch_one(const CUtensorMap& W0, const CUtensorMap& W1, const CUtensorMap& S0,
                              const CUtensorMap& S1, const CUtensorMap& X, const StreamParams& p, int grid,
                              int smem, bool pdl, cudaStream_t s) {
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(stream_kernel<MODE, FOLD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             FOLD ? kFoldMaxSmem : SCfg<MODE, FOLD>::SMEM);
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    {
        ProfScope prof_(MODE == 0 ? MOE_K_STREAM_GATEUP : MOE_K_STREAM_DOWN, s);
        const cudaError_t le = launch_pdl(pdl, stream_kernel<MODE, FOLD>, dim3(grid), dim3(THREADS), smem, s, W0,
                                          W1, S0, S1, X, p);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace st

// Gate/up (+ reduce) then down for the experts on the streaming list.
// xg: the gathered rows [rows, d] (bf16); h: [rows, f] fp16.
cudaError_t launch_stream_ffn(const Dims& D, const uint16_t* xg, uint16_t* h, float* part, const int32_t* offsets,
                              const int32_t* stream_list, const int32_t* n_stream, const int32_t* sorted_pair,
                              const float* topk_w, const moe_weights* w, uint16_t* y_rows, uint32_t* err,
                              uint64_t wait_ns, const CombineArgs* comb, cudaStream_t s) {
    using namespace st;
    CUtensorMap mG, mU, mD, mSG, mSU, mSD, mX, mH;
    if (!map_2d(&mG, w->w_gate, int64_t(D.E) * D.d, D.f, BKS) || !map_2d(&mU, w->w_up, int64_t(D.E) * D.d, D.f, BKS) ||
        !map_chunks(&mD, w->w_down, int64_t(D.E) * D.f, D.d, 4) || !map_2d(&mX, xg, D.rows, D.d, RC) ||
        !map_2d(&mH, h, D.rows, D.f, RC))
        return cudaErrorInvalidValue;
    if (D.has_shared) {
        if (!map_2d(&mSG, w->shared_gate, D.d, D.f, BKS) || !map_2d(&mSU, w->shared_up, D.d, D.f, BKS) ||
            !map_chunks(&mSD, w->shared_down, D.f, D.d, 4))
            return cudaErrorInvalidValue;
    } else {
        mSG = mG;
        mSU = mU;
        mSD = mD;
    }
    const int grid = num_sms();
    StreamParams p{};
    p.E = D.E;
    p.etot = D.Etot;
    p.offsets = offsets;
    p.stream_list = stream_list;
    p.n_stream = n_stream;
    p.sorted_pair = sorted_pair;
    p.topk_w = topk_w;
    p.rows = D.rows;
    p.limit = D.limit;
    p.down_f16 = D.down_f16;
    p.err = err;
    p.wait_ns = wait_ns;
    // gate/up
    p.mode = 0;
    p.K = D.d;
    p.N = D.f;
    p.ks = D.ks;
    p.kslice = D.d / D.ks;
    p.out = h;
    p.part = part;
    const bool pdl = use_pdl(D.T);
    cudaError_t e = launch_one<0>(mG, mU, mSG, mSU, mX, p, grid, SCfg<0>::SMEM, pdl, s);
    if (e != cudaSuccess) return e;
    const bool fold = stream_fold(D);
    if (D.ks > 1 && !fold) {
        ProfScope prof_(MOE_K_STREAM_REDUCE, s);
        const cudaError_t le = launch_pdl(pdl, stream_reduce_kernel, dim3(grid * 2), dim3(256), 0, s, part, D.ks,
                                          D.rows, D.f, offsets, stream_list, n_stream, D.limit, h, err);
        if (le != cudaSuccess) return le;
    }
    // down
    p.mode = 1;
    p.K = D.f;
    p.N = D.d;
    p.ks = 1;
    p.kslice = D.f;
    p.out = y_rows;
    p.part = nullptr;
    if (comb) {
        p.comb_count = comb->count;
        p.pair_row = comb->pair_row;
        p.comb_out = comb->out;
        p.comb_bf16 = D.out_bf16;
        p.T = D.T;
        p.k = D.k;
        p.has_shared = D.has_shared;
    }
    if (fold) {
        p.hpart = part;
        p.ksg = D.ks;
        return launch_one<1, true>(mD, mD, mSD, mSD, mH, p, grid, SCfg<1, true>::SMEM + RC * fold_row_bytes(D.f),
                                   pdl, s);
    }
    return launch_one<1>(mD, mD, mSD, mSD, mH, p, grid, SCfg<1>::SMEM, pdl, s);
}

// The streaming down kernel sums the K-split gate/up partials itself (no reduce
// kernel) when its h buffer of RC rows fits beside its stages.
bool stream_fold(const Dims& D) { return D.ks > 1 && D.ks <= st::kFoldMaxSlices && st::fold_fits(D.f); }

}  // namespace moe

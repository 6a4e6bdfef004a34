// gemm_tc.cu — S5, S6 (+ S9) on the 5th-generation tensor cores: one
// persistent grouped GEMM kernel, one SM per tile, used twice per layer:
//   MODE 0: h = silu(clamp(x W_gate[e])) * clamp(x W_up[e])   (S5, SwiGLU fused)
//   MODE 1: y = w_pair * (h W_down[e])                          (S6, gate scale fused)
// with the weights either bf16 ([E, K, N], N contiguous) or Q4G32 (4-bit,
// dequantised in the kernel once per weight tile: S9).
//
// Prior art: "Strata PR #4366" (DS4_FAT_ROWS), Approach — a popular expert's
// packed weights decoded once to FP16, its rows gathered, one FP16 GEMM, then a
// clamped SwiGLU in FP16; "mini-AGI PR #4" run() — experts grouped by load,
// each group at its own size. Here every expert with rows becomes
// ceil(rows/128) M-tiles of one grouped launch; rows past an expert's end are
// computed and masked.
//
// Kernel shape (one CTA per SM, persistent over work units):
//   warp 0    TMA producer. A = 128 rows x 64 K of the gathered rows (2-D map,
//             128-byte swizzle, K-major), two such sub-tiles for 256-row units.
//             B, bf16: 64 K x 256 N of the expert's weights (3-D map, four
//             64-wide boxes, N-major). B, Q4G32: the packed nibbles of 256
//             N-rows x 64 K (32 bytes a row) and the k-block's two scale groups.
//   warp 1    TMEM allocator + single-thread tcgen05.mma issuer: M=128, N=256,
//             K=16 per instruction, fp32 accumulators in TMEM. bf16 units are
//             128 rows with two 256-column buffers, so the epilogue of a unit
//             overlaps the next unit's MMAs; Q4G32 units are 256 rows (two
//             M=128 MMAs per B tile, one buffer of 2 x 256 columns), halving
//             the dequantisation per FLOP.
//   warps 2-5 epilogue: tcgen05.ld 32 lanes x 32 columns, fused SwiGLU or gate
//             scaling, fp16 stores. Warp w reads TMEM lanes 32*(w%4)..+31.
//   warps 6.. transform (8 for Q4G32, 4 for MODE 1 with W_down given as bf16): turn the
//             landed B tile into fp16 — bf16 -> fp16 in place (costly: it
//             competes with the MMA for shared-memory bandwidth, so W_down is
//             normally prepared as fp16 once at load time and this is skipped),
//             or nibbles x scale -> fp16 written in the
//             K-major 128-byte-swizzled layout the MMA reads — then release it
//             to the MMA warp (generic-proxy writes fenced for the async proxy).
// Operand types per MMA: MODE 0 bf16 x bf16 (fp16 x fp16 with Q4G32, x being
// gathered as fp16); MODE 1 fp16 x fp16 (h is fp16). fp32 accumulate always.
// A work unit is (expert, n-tile, m-tile); units of one expert and n-tile are
// adjacent so its weight tile is read from HBM once and served from L2 to its
// other M-tiles. Every mbarrier wait is bounded in time; a wait that gives up
// raises MOE_DEVERR_TIMEOUT, the CTA drains its copies and MMAs, frees TMEM and
// returns. Every TMA copy fills only the issuing CTA's shared memory.
#include "gemm_tc.cuh"

namespace moe {

namespace tc {

// WF: weight form. 0 = bf16 as given, 1 = Q4G32, 2 = fp16 (W_down prepared at load time).
// GATHER (bf16 gate/up, one SM per 128-row tile only): four gather warps copy the
// A rows straight from x (cp.async, 16 bytes a lane, into the 128-byte-swizzled
// tile) instead of TMA loads of a gathered copy.
template <int MODE, int WF, int SUB, bool GATHER = false>
struct Cfg {
    static constexpr bool Q4 = WF == 1;
    static constexpr bool kTransform = Q4 || (MODE == 1 && WF == 0);
    // Rows of a unit, in 128-row sub-tiles (SUB = 1 or 2). With SUB = 2 two
    // M=128 MMAs share every B tile, so B is loaded (and for Q4G32
    // dequantised) once per 256 rows; the two accumulators then fill TMEM and
    // there is one accumulator buffer instead of two, so the epilogue is not
    // overlapped with the next unit's MMAs. Measured on B200: SUB = 2 pays for
    // the Q4G32 GEMMs (dequantisation halves per FLOP), SUB = 1 for bf16.
    static constexpr int kSub = SUB;
    static constexpr int kAcc = 2 / kSub;  // accumulator buffers of kSub x 256 columns
    static constexpr int kEpiWarps = 4;
    // transform warps: 8 for Q4G32 (the dequantisation sits between the copy and
    // the MMA of every stage; measured 2% faster than 4), 4 for the bf16 -> fp16 pass
    static constexpr int kTransWarps = kTransform ? (Q4 ? 8 : 4) : 0;
    static constexpr int kGatherWarps = GATHER ? 4 : 0;
    static_assert(!GATHER || (MODE == 0 && WF == 0 && SUB == 1), "gather warps: bf16 gate/up, 128-row units");
    static constexpr int kThreads = 32 * (2 + kEpiWarps + kTransWarps + kGatherWarps);
    static constexpr int kABytes = kSub * A_BYTES;
    static constexpr int kStages = (Q4 || kSub == 2) ? 3 : 4;
    static constexpr int kStageBytes = Q4 ? kABytes + B_BYTES + P_BYTES + S_BYTES : kABytes + B_BYTES;
    // bytes a stage receives besides its A sub-tiles (A_BYTES each)
    static constexpr uint32_t kTxB = Q4 ? P_BYTES + S_BYTES : B_BYTES;
    static constexpr int kSmem = 1024 + kStages * kStageBytes + 512;  // + barriers, unit ring
    // warps that read the unit ring: MMA, epilogue, transform, gather
    static constexpr int kUnitReaders = 1 + kEpiWarps + kTransWarps + kGatherWarps;
    // bf16 operands for the bf16 gate/up; fp16 otherwise. B is N-major (bf16
    // weights as stored) or K-major (dequantised from the K-major Q4G32 rows).
    static constexpr uint32_t kIdesc =
        idesc_f16_f32(BM, BN, /*ab_bf16=*/(MODE == 0 && WF == 0) ? 1 : 0, /*a_mn=*/0, /*b_mn=*/Q4 ? 0 : 1);
    // An expert's last tile with <= 64 rows runs M=64 (half the MMA work). Its
    // accumulator sits in lanes 0-15 of each 32-lane TMEM sub-partition: row m
    // in lane 32*(m/16) + m%16, every column as for M=128.
    static constexpr uint32_t kIdesc64 =
        idesc_f16_f32(64, BN, /*ab_bf16=*/(MODE == 0 && WF == 0) ? 1 : 0, /*a_mn=*/0, /*b_mn=*/Q4 ? 0 : 1);
};

MOE_DEV uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t orv) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(orv));  // (a & b) | c
    return r;
}
MOE_DEV uint32_t hsub2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
MOE_DEV uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// One Q4G32 word (k = 8i..8i+7, nibble p holding k 8i+{0,2,4,6,1,3,5,7}[p])
// times its scale pair -> eight fp16 in k order. (w >> 4j) & 0x000F000F keeps
// nibbles j and j+4, i.e. k = 2j and 2j+1; OR-ing 0x6400 makes each the fp16
// value 1024 + u exactly, minus 1032 gives q = u - 8 exactly, then one rounding
// for q * s.
MOE_DEV uint4 dequant_word(uint32_t w, uint32_t s2) {
    constexpr uint32_t kMask = 0x000F000Fu, kMagic = 0x64006400u, kBias = 0x64086408u;
    uint4 o;
    o.x = hmul2(hsub2(lop3_and_or(w, kMask, kMagic), kBias), s2);
    o.y = hmul2(hsub2(lop3_and_or(w >> 4, kMask, kMagic), kBias), s2);
    o.z = hmul2(hsub2(lop3_and_or(w >> 8, kMask, kMagic), kBias), s2);
    o.w = hmul2(hsub2(lop3_and_or(w >> 12, kMask, kMagic), kBias), s2);
    return o;
}


template <int MODE, int WF, int SUB, bool GATHER = false>
__global__ void __launch_bounds__(Cfg<MODE, WF, SUB, GATHER>::kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmS0,
                        const __grid_constant__ CUtensorMap tmS1, const GemmParams p) {
    using C = Cfg<MODE, WF, SUB, GATHER>;
    constexpr bool Q4 = C::Q4;
    constexpr int STAGES = C::kStages, SB = C::kStageBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * SB);
    uint64_t* conv = full + STAGES;  // B tile transformed (fp16) and ready for the MMA
    uint64_t* empty = conv + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint64_t* ufull = drain + 1;  // unit ring: slot holds the next claimed unit
    uint64_t* uempty = ufull + UR;
    volatile int* unit_ring = reinterpret_cast<volatile int*>(uempty + UR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(unit_ring) + UR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1 + C::kGatherWarps);  // the producer's byte count (+ one arrival per gather warp)
            mbar_init(conv + s, 32 * C::kTransWarps);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, C::kEpiWarps);
        }
        for (int r = 0; r < UR; ++r) {
            mbar_init(ufull + r, 1);
            mbar_init(uempty + r, C::kUnitReaders);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB0);
        tma_prefetch_desc(&tmB1);
        if (Q4) {
            tma_prefetch_desc(&tmS0);
            tma_prefetch_desc(&tmS1);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // the prologue above touched no global memory; wait for the predecessor here
    griddep_wait();
    griddep_launch();

    const int nt = p.n_tiles;
    const int total_units = __ldg(p.tile_base + p.Etot) * nt;
    const int KB = p.K / BK;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        int stage = 0;
        uint32_t phase = 0, issued = 0, issued_par = 0;
        bool ok = true;
        int uslot = 0;
        uint32_t uphase = 0;
        while (ok) {
            int u = -1;
            if (!ring_publish(u, uslot, uphase, p.unit_counter, total_units, unit_ring, ufull, uempty, abort_flag, p.err,
                              p.wait_ns)) {
                ok = false;
                break;
            }
            if (u < 0) break;
            const Unit U = decode_unit<C::kSub>(u, p, nt);
            const bool sh = U.e >= p.E;
            const int z = sh ? 0 : U.e;
            for (int kb = 0; kb < KB; ++kb) {
                int okl = 1;
                if (lane == 0) okl = mbar_wait_bounded(empty + stage, phase ^ 1u, abort_flag, p.err, p.wait_ns);
                okl = __shfl_sync(0xFFFFFFFFu, okl, 0);
                if (!okl) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    uint8_t* sa = smem + stage * SB;
                    uint8_t* sb = sa + C::kABytes;
                    const bool a1 = C::kSub == 2 && U.rows > BM;  // second 128-row sub-tile present
                    mbar_arrive_expect_tx(full + stage, C::kTxB + (GATHER ? 0u : (a1 ? 2u : 1u) * A_BYTES));
                    if (!GATHER) tma_load_2d(sa, &tmA, full + stage, kb * BK, U.row0);
                    if (a1) tma_load_2d(sa + A_BYTES, &tmA, full + stage, kb * BK, U.row0 + BM);
                    if (Q4) {
                        // packed rows [N][32 B] and scales [2 groups][rows] fp16
                        uint8_t* sp = sb + B_BYTES;
                        uint8_t* ss = sp + P_BYTES;
                        if (MODE == 0) {
                            const int n0 = U.n * 128;
                            tma_load_3d(sp, &tmB0, full + stage, kb * (BK / 2), n0, z);
                            tma_load_3d(sp + P_BYTES / 2, &tmB1, full + stage, kb * (BK / 2), n0, z);
                            tma_load_3d(ss, &tmS0, full + stage, n0, kb * 2, z);
                            tma_load_3d(ss + S_BYTES / 2, &tmS1, full + stage, n0, kb * 2, z);
                        } else {
                            const int n0 = U.n * BN;
                            tma_load_3d(sp, &tmB0, full + stage, kb * (BK / 2), n0, z);
                            tma_load_3d(ss, &tmS0, full + stage, n0, kb * 2, z);
                        }
                    } else if (MODE == 0) {
                        const CUtensorMap* mg = sh ? &tmS0 : &tmB0;
                        const CUtensorMap* mu = sh ? &tmS1 : &tmB1;
                        // two 64-column chunks of gate, then two of up: one copy each
                        tma_load_4d(sb, mg, full + stage, 0, kb * BK, 2 * U.n, z);
                        tma_load_4d(sb + 2 * B_CHUNK, mu, full + stage, 0, kb * BK, 2 * U.n, z);
                    } else {
                        const CUtensorMap* md = sh ? &tmS0 : &tmB0;
                        // four 64-column chunks in one copy
                        tma_load_4d(sb, md, full + stage, 0, kb * BK, 4 * U.n, z);
                    }
                    issued |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                }
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // On abort, let every copy already issued land before the CTA can exit.
        if (!ok && lane == 0) {
            for (int s = 0; s < STAGES; ++s)
                if (issued >> s & 1u) mbar_wait_bounded(full + s, (issued_par >> s) & 1u, nullptr, p.err, kDrainLimitNs);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t IDESC = C::kIdesc;
        uint64_t* ready = C::kTransform ? conv : full;
        int stage = 0, acc = 0;
        uint32_t phase = 0, acc_phase = 0;
        bool ok = true;
        int uslot = 0;
        uint32_t uphase = 0;
        while (ok) {
            int u = -1;
            if (!ring_read(u, uslot, uphase, unit_ring, ufull, uempty, abort_flag, p.err, p.wait_ns)) break;
            if (u < 0) break;
            int okl = 1;
            if (lane == 0) okl = mbar_wait_bounded(tempty + acc, acc_phase ^ 1u, abort_flag, p.err, p.wait_ns);
            okl = __shfl_sync(0xFFFFFFFFu, okl, 0);
            if (!okl) break;
            tc_fence_after();
            const int rows = decode_unit<C::kSub>(u, p, nt).rows;
            const uint32_t d_tmem = tmem_base + uint32_t(acc * C::kSub * BN);
            const bool m64 = min(rows, BM) <= 64;
            const uint32_t idesc = m64 ? C::kIdesc64 : IDESC;
            // second sub-tile (rows 128..255 of the unit), its accumulator 256 columns on
            const bool sub1 = C::kSub == 2 && rows > BM;
            const uint32_t idesc1 = rows - BM <= 64 ? C::kIdesc64 : IDESC;
            for (int kb = 0; kb < KB; ++kb) {
                if (lane == 0) okl = mbar_wait_bounded(ready + stage, phase, abort_flag, p.err, p.wait_ns);
                okl = __shfl_sync(0xFFFFFFFFu, okl, 0);
                if (!okl) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t a0 = smem_u32(smem + stage * SB);
                    const uint32_t b0 = a0 + C::kABytes;
#pragma unroll
                    for (int j = 0; j < BK / 16; ++j) {
                        // A: K-major, advance 16 elements = 32 bytes inside the swizzle row.
                        // B: N-major (bf16 weights): advance 16 K-rows = 2 KB;
                        //    K-major (dequantised Q4G32): like A.
                        const uint64_t ad = sdesc_sw128(a0 + j * 32, 16, 1024);
                        const uint64_t bd = Q4 ? sdesc_sw128(b0 + j * 32, 16, 1024)
                                               : sdesc_sw128(b0 + j * 2048, B_CHUNK, 1024);
                        umma_bf16(d_tmem, ad, bd, idesc, (kb | j) != 0);
                        if (sub1)
                            umma_bf16(d_tmem + BN, sdesc_sw128(a0 + A_BYTES + j * 32, 16, 1024), bd, idesc1,
                                      (kb | j) != 0);
                    }
                    umma_commit(empty + stage);
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) umma_commit(tfull + acc);
            __syncwarp();
            if (++acc == C::kAcc) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        // every MMA this thread issued has completed before TMEM is freed
        if (lane == 0) {
            umma_commit(drain);
            mbar_wait_bounded(drain, 0, nullptr, p.err, kDrainLimitNs);
        }
        __syncwarp();
    } else if (warp < 2 + C::kEpiWarps) {
        // ------------------------------------------------ epilogue (warps 2 .. 2+kEpiWarps-1)
        // Warp w reads TMEM lanes 32*(w%4) .. +31, for each sub-tile in turn.
        const int q = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool range_bad = false;
        int uslot = 0;
        uint32_t uphase = 0;
        while (true) {
            int u = -1;
            if (!ring_read(u, uslot, uphase, unit_ring, ufull, uempty, abort_flag, p.err, p.wait_ns)) break;
            if (u < 0) break;
            const Unit U = decode_unit<C::kSub>(u, p, nt);
            int okl = 1;
            if (lane == 0) okl = mbar_wait_bounded(tfull + acc, acc_phase, abort_flag, p.err, p.wait_ns);
            okl = __shfl_sync(0xFFFFFFFFu, okl, 0);
            if (!okl) break;
            tc_fence_after();
#pragma unroll 1
            for (int sub = 0; sub < C::kSub; ++sub) {
                const int rows = min(BM, U.rows - sub * BM);
                if (rows <= 0) break;
                const uint32_t tb = tmem_base + (uint32_t(q * 32) << 16) + uint32_t((acc * C::kSub + sub) * BN);
                epilogue_tile<MODE>(tb, U.n, int64_t(U.row0) + sub * BM, rows, rows <= 64, q, lane, p, range_bad);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty + acc);
            if (++acc == C::kAcc) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (range_bad) set_error(p.err, MOE_DEVERR_RANGE);
    } else if (GATHER) {
        // ------------------------------------------------ gather (the last 4 warps)
        // Warp gw copies tile rows 32gw..32gw+31: lane = (row 4i + lane/8 of the
        // warp's 32, 16-byte chunk lane%8 of the row's 128 bytes), so one
        // instruction moves four whole 128-byte rows. A stage is released to
        // the MMA one stage later: after the next stage's copies are issued,
        // wait for the older group, make it visible to the tensor core (proxy
        // fence) and arrive on its full barrier. Rows past the unit's end are
        // zero-filled.
        const int gw = warp - (2 + C::kEpiWarps);
        const int cch = lane & 7;
        int stage = 0, prev = -1;
        uint32_t phase = 0;
        bool ok = true;
        int uslot = 0;
        uint32_t uphase = 0;
        bool bad = false;
        while (ok) {
            int u = -1;
            if (!ring_read(u, uslot, uphase, unit_ring, ufull, uempty, abort_flag, p.err, p.wait_ns)) break;
            if (u < 0) break;
            const Unit U = decode_unit<1>(u, p, nt);
            const uint16_t* src[8];
            uint32_t nbytes[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = 32 * gw + 4 * i + (lane >> 3);
                src[i] = p.x;
                nbytes[i] = 0;
                if (r < U.rows) {
                    const int t = __ldg(p.sorted_token + U.row0 + r);
                    if (t >= 0 && t < p.T) {
                        src[i] = p.x + int64_t(t) * p.K + cch * 8;
                        nbytes[i] = 16;
                    } else {
                        bad = true;
                    }
                }
            }
            for (int kb = 0; kb < KB; ++kb) {
                int okl = 1;
                if (lane == 0) okl = mbar_wait_bounded(empty + stage, phase ^ 1u, abort_flag, p.err, p.wait_ns);
                okl = __shfl_sync(0xFFFFFFFFu, okl, 0);
                if (!okl) {
                    ok = false;
                    break;
                }
                const uint32_t sa = smem_u32(smem + stage * SB);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 32 * gw + 4 * i + (lane >> 3);
                    cp_async_16(sa + r * 128 + ((cch ^ (r & 7)) << 4), src[i] + kb * BK, nbytes[i]);
                }
                cp_async_commit();
                if (prev >= 0) {
                    cp_async_wait<1>();
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(full + prev);
                }
                prev = stage;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // the last stage (or, after an abort, every copy in flight) lands before exit
        cp_async_wait<0>();
        fence_proxy_async_smem();
        __syncwarp();
        if (ok && prev >= 0 && lane == 0) mbar_arrive(full + prev);
        if (bad) set_error(p.err, MOE_DEVERR_BOUNDS);
    } else if (C::kTransform) {
        // ------------------------------------------------ transform (the last kTransWarps warps)
        const int ct = threadIdx.x - 32 * (2 + C::kEpiWarps);  // 0 .. 32*kTransWarps-1
        constexpr int NT = 32 * C::kTransWarps;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int uslot = 0;
        uint32_t uphase = 0;
        while (ok) {
            int u = -1;
            if (!ring_read(u, uslot, uphase, unit_ring, ufull, uempty, abort_flag, p.err, p.wait_ns)) break;
            if (u < 0) break;
            for (int kb = 0; kb < KB; ++kb) {
                int okl = 1;
                if (lane == 0) okl = mbar_wait_bounded(full + stage, phase, abort_flag, p.err, p.wait_ns);
                okl = __shfl_sync(0xFFFFFFFFu, okl, 0);
                if (!okl) {
                    ok = false;
                    break;
                }
                uint8_t* sb = smem + stage * SB + C::kABytes;
                if (Q4) {
                    // 512 (row, half) pairs of the 256-row B tile, 512/NT per thread;
                    // half hf of row r is words 4hf..4hf+3 (k 32hf..32hf+31, scale
                    // group hf) -> chunks 4hf+c of 8 fp16 at r*128 + (((4hf+c) ^ (r%8)) * 16).
                    // Consecutive lanes read consecutive 16-byte words (no bank conflicts).
                    const uint8_t* sp = sb + B_BYTES;
                    const uint16_t* ss = reinterpret_cast<const uint16_t*>(sp + P_BYTES);
#pragma unroll
                    for (int it = 0; it < 512 / NT; ++it) {
                        const int q = ct + NT * it;
                        const int r = q >> 1, hf = q & 1;
                        // scales [2 groups][rows]: MODE 0 holds gate rows then up rows (128 each)
                        const uint32_t sc = MODE == 0 ? ss[(r >> 7) * 256 + hf * 128 + (r & 127)] : ss[hf * 256 + r];
                        const uint32_t s2 = sc | (sc << 16);
                        const uint4 w = reinterpret_cast<const uint4*>(sp + r * 32)[hf];
                        const uint32_t words[4] = {w.x, w.y, w.z, w.w};
                        uint8_t* row = sb + r * 128;
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            *reinterpret_cast<uint4*>(row + (((4 * hf + c) ^ (r & 7)) << 4)) = dequant_word(words[c], s2);
                    }
                } else {
                    // bf16 -> fp16 in place (position-independent)
                    uint4* b = reinterpret_cast<uint4*>(sb);
#pragma unroll 4
                    for (int i = ct; i < B_BYTES / 16; i += NT) {
                        uint4 v = b[i];
                        v.x = bf16x2_to_f16x2(v.x);
                        v.y = bf16x2_to_f16x2(v.y);
                        v.z = bf16x2_to_f16x2(v.z);
                        v.w = bf16x2_to_f16x2(v.w);
                        b[i] = v;
                    }
                }
                fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
                mbar_arrive(conv + stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace tc

// ---------------------------------------------------------------------------- host side

namespace tc {

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

// dims/strides innermost first (strides in bytes, rank-1 of them).
static bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz) {
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    if (rank < 1 || rank > 5) return false;
    cuuint64_t gd[5], gs[4];
    cuuint32_t bx[5], es[5] = {1, 1, 1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        gd[i] = dims[i];
        bx[i] = box[i];
    }
    for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
    const CUresult r = enc(m, dt, rank, const_cast<void*>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// A operand: rows x K 2-byte elements, row-major; box 64 (K) x 128 (rows), 128-byte swizzle.
bool map_rows(CUtensorMap* m, const void* base, int64_t rows, int K) {
    const uint64_t dims[2] = {uint64_t(K), uint64_t(rows)};
    const uint64_t str[1] = {uint64_t(K) * 2};
    const uint32_t box[2] = {64, 128};
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}
// bf16 B operand: [nexp, K, N] row-major, seen as [nexp, N/64 chunks, K, 64] so that one
// copy brings `chunks` 64-column boxes of 64 K-rows (128-byte swizzle), stored chunk after
// chunk (8 KB apart) — fewer copies for the single producer thread to issue.
bool map_weights(CUtensorMap* m, const void* base, int nexp, int K, int N, int chunks) {
    const uint64_t dims[4] = {64, uint64_t(K), uint64_t(N / 64), uint64_t(nexp)};
    const uint64_t str[3] = {uint64_t(N) * 2, 128, uint64_t(N) * uint64_t(K) * 2};
    const uint32_t box[4] = {64, 64, uint32_t(chunks), 1};
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}
// 2-byte weights [nexp, N, K] (K contiguous) read as a K-major B operand: box 64 (K)
// x 256 (N rows) x 1, 128-byte swizzle — the layout of the A tiles, 256 rows.
bool map_weights_kmajor(CUtensorMap* m, const void* base, int nexp, int N, int K, bool f16) {
    const uint64_t dims[3] = {uint64_t(K), uint64_t(N), uint64_t(nexp)};
    const uint64_t str[2] = {uint64_t(K) * 2, uint64_t(N) * uint64_t(K) * 2};
    const uint32_t box[3] = {64, 256, 1};
    return make_map(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 3, dims, str,
                    box, CU_TENSOR_MAP_SWIZZLE_128B);
}
// 2-byte activation rows [rows, N] (row stride row_stride elements) read as an N-major
// operand with K = rows: seen as [1, N/64 chunks, rows, 64]; one copy brings `chunks`
// 64-column chunks of 64 K-rows (4 for a 256-wide B, 2 for a 128-wide A).
bool map_act_mn(CUtensorMap* m, const void* base, int64_t rows, int N, int64_t row_stride, int chunks) {
    const uint64_t dims[4] = {64, uint64_t(rows), uint64_t(N / 64), 1};
    const uint64_t str[3] = {uint64_t(row_stride) * 2, 128, uint64_t(row_stride) * uint64_t(rows) * 2};
    const uint32_t box[4] = {64, 64, uint32_t(chunks), 1};
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 4, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}
// 2-byte rows [rows, cols] (bf16 or fp16) written by 32 x 32 boxes (64-byte swizzle)
// from shared memory.
bool map_rows_store32(CUtensorMap* m, const void* base, int64_t rows, int cols, bool f16) {
    const uint64_t dims[2] = {uint64_t(cols), uint64_t(rows)};
    const uint64_t str[1] = {uint64_t(cols) * 2};
    const uint32_t box[2] = {32, 32};
    return make_map(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, 2, dims, str,
                    box, CU_TENSOR_MAP_SWIZZLE_64B);
}
// fp32 [nexp, M, N] written by 32 x 32 boxes (128-byte swizzle) from shared memory.
bool map_f32_tiles(CUtensorMap* m, const void* base, int nexp, int M, int N) {
    const uint64_t dims[3] = {uint64_t(N), uint64_t(M), uint64_t(nexp)};
    const uint64_t str[2] = {uint64_t(N) * 4, uint64_t(M) * uint64_t(N) * 4};
    const uint32_t box[3] = {32, 32, 1};
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}
// Q4G32 nibbles: [nexp, N, K/2] bytes; box 32 bytes (64 k) x rows x 1, no swizzle.
bool map_q4_packed(CUtensorMap* m, const void* base, int nexp, int K, int N, int rows) {
    const uint64_t dims[3] = {uint64_t(K / 2), uint64_t(N), uint64_t(nexp)};
    const uint64_t str[2] = {uint64_t(K / 2), uint64_t(N) * uint64_t(K / 2)};
    const uint32_t box[3] = {32, uint32_t(rows), 1};
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}
// Q4G32 scales: [nexp, K/32, N] fp16; box rows (N) x 2 groups x 1, no swizzle.
bool map_q4_scales(CUtensorMap* m, const void* base, int nexp, int K, int N, int rows) {
    const uint64_t dims[3] = {uint64_t(N), uint64_t(K / 32), uint64_t(nexp)};
    const uint64_t str[2] = {uint64_t(N) * 2, uint64_t(N) * uint64_t(K / 32) * 2};
    const uint32_t box[3] = {uint32_t(rows), 2, 1};
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, base, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <int MODE, int WF, int SUB, bool GATHER = false>
cudaError_t launch_gemm(const CUtensorMap& A, const CUtensorMap& B0, const CUtensorMap& B1, const CUtensorMap& S0,
                        const CUtensorMap& S1, const GemmParams& p, bool pdl, cudaStream_t s) {
    using C = Cfg<MODE, WF, SUB, GATHER>;
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<MODE, WF, SUB, GATHER>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    GemmParams q = p;
    if (C::kSub == 2) q.tile_base = p.tile_base + p.Etot + 1;  // 256-row units
    {
        ProfScope prof_(MODE == 0 ? MOE_K_TC_GATEUP : MOE_K_TC_DOWN, s);
        const cudaError_t le = launch_pdl(pdl, grouped_gemm_kernel<MODE, WF, SUB, GATHER>, dim3(num_sms()), dim3(C::kThreads),
                                          C::kSmem, s, A, B0, B1, S0, S1, q);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace tc

// Both tcgen05 GEMMs of the tile variant. xg: the gathered rows (bf16, or
// fp16 for Q4G32); h: [rows, f] fp16 scratch.
cudaError_t launch_tensor_ffn(const Dims& D, const uint16_t* xg, uint16_t* h, const int32_t* tile_base,
                              const int32_t* offsets,
                              const int32_t* sorted_pair, const float* topk_w, const moe_weights* w,
                              uint16_t* y_rows, int32_t* counters, uint32_t* err, uint64_t wait_ns,
                              const uint16_t* x_fused, const int32_t* sorted_token, cudaStream_t s) {
    using namespace tc;
    const bool pdl = use_pdl(D.T);
    GemmParams p{};
    p.E = D.E;
    p.Etot = D.Etot;
    p.tile_base = tile_base;
    p.offsets = offsets;
    p.sorted_pair = sorted_pair;
    p.topk_w = topk_w;
    p.limit = D.limit;
    p.err = err;
    p.wait_ns = wait_ns;
    CUtensorMap mA, mH;
    if (!map_rows(&mA, xg, D.rows, D.d) || !map_rows(&mH, h, D.rows, D.f)) return cudaErrorInvalidValue;
    cudaError_t e;
    if (D.fmt == MOE_WEIGHTS_Q4G32) {
        CUtensorMap pg, pu, sg, su, pd, sd;
        if (!map_q4_packed(&pg, w->w_gate, D.E, D.d, D.f, 128) || !map_q4_packed(&pu, w->w_up, D.E, D.d, D.f, 128) ||
            !map_q4_scales(&sg, w->s_gate, D.E, D.d, D.f, 128) || !map_q4_scales(&su, w->s_up, D.E, D.d, D.f, 128) ||
            !map_q4_packed(&pd, w->w_down, D.E, D.f, D.d, BN) || !map_q4_scales(&sd, w->s_down, D.E, D.f, D.d, BN))
            return cudaErrorInvalidValue;
        p.K = D.d;
        p.n_out = D.f;
        p.n_tiles = (D.f + 127) / 128;
        p.out = h;
        p.unit_counter = counters;
        if ((e = launch_gemm<0, 1, 2>(mA, pg, pu, sg, su, p, pdl, s)) != cudaSuccess) return e;
        p.K = D.f;
        p.n_out = D.d;
        p.n_tiles = (D.d + BN - 1) / BN;
        p.out = y_rows;
        p.unit_counter = counters + 1;
        return launch_gemm<1, 1, 2>(mH, pd, pd, sd, sd, p, pdl, s);
    }
    CUtensorMap mG, mU, mSG, mSU, mD, mSD;
    if (!map_weights(&mG, w->w_gate, D.E, D.d, D.f, 2) || !map_weights(&mU, w->w_up, D.E, D.d, D.f, 2) ||
        !map_weights(&mD, w->w_down, D.E, D.f, D.d, 4))
        return cudaErrorInvalidValue;
    if (D.has_shared) {
        if (!map_weights(&mSG, w->shared_gate, 1, D.d, D.f, 2) || !map_weights(&mSU, w->shared_up, 1, D.d, D.f, 2) ||
            !map_weights(&mSD, w->shared_down, 1, D.f, D.d, 4))
            return cudaErrorInvalidValue;
    } else {
        mSG = mG;
        mSU = mU;
        mSD = mD;
    }
    // S5: gate/up + SwiGLU -> h (the gate/up maps bring 2 chunks a copy: the
    // one-SM kernel copies gate and up, each SM of a pair one of them)
    p.K = D.d;
    p.n_out = D.f;
    p.n_tiles = (D.f + 127) / 128;
    p.out = h;
    p.unit_counter = counters;
    p.x = x_fused;
    p.sorted_token = sorted_token;
    p.T = D.T;
    e = D.tile_pair ? launch_gemm_pair<0>(mA, mG, mU, mSG, mSU, p, pdl, s)
        : x_fused   ? launch_gemm<0, 0, 1, true>(mA, mG, mU, mSG, mSU, p, pdl, s)
                    : launch_gemm<0, 0, 1>(mA, mG, mU, mSG, mSU, p, pdl, s);
    if (e != cudaSuccess) return e;
    // S6: down + gate scale -> y_rows
    p.K = D.f;
    p.n_out = D.d;
    p.n_tiles = (D.d + BN - 1) / BN;
    p.out = y_rows;
    p.unit_counter = counters + 1;
    if (D.tile_pair && D.down_f16) {
        // each SM of a pair copies 128 of the tile's 256 columns: maps of 2 chunks
        CUtensorMap mD2, mSD2;
        if (!map_weights(&mD2, w->w_down, D.E, D.f, D.d, 2)) return cudaErrorInvalidValue;
        if (D.has_shared) {
            if (!map_weights(&mSD2, w->shared_down, 1, D.f, D.d, 2)) return cudaErrorInvalidValue;
        } else {
            mSD2 = mD2;
        }
        return launch_gemm_pair<1>(mH, mD2, mD2, mSD2, mSD2, p, pdl, s);
    }
    return D.down_f16 ? launch_gemm<1, 2, 1>(mH, mD, mD, mSD, mSD, p, pdl, s)
                      : launch_gemm<1, 0, 1>(mH, mD, mD, mSD, mSD, p, pdl, s);
}

}  // namespace moe

// gemm_pair.cu — S5 and S6 on SM pairs: the grouped GEMMs of gemm_tc.cu with
// tcgen05 ops of cta_group::2, for bf16 gate/up weights (MODE 0, SwiGLU fused)
// and W_down prepared as fp16 (MODE 1, gate scale fused).
//
// Why pairs. With one SM per 128 x 256 tile, every k-block of 64 brings 48 KB
// into the SM (16 KB of rows, 32 KB of weights) for 4.2 MFLOP. Two SMs of a
// cluster computing one 256 x 256 tile each bring their own 128 rows and half
// of the 256 weight columns, 32 KB for the same 4.2 MFLOP per SM: a third less
// L2-to-SM traffic per FLOP, and six 32 KB stages in flight instead of four of
// 48 KB. The cost is rounding experts up to 256 rows instead of 128 (the rows
// past an expert's end are computed and masked), so the pair kernels are used
// when experts average at least 256 rows.
//
// Roles (rank 0 of the cluster is the leader, rank 1 the peer):
//   warp 0    TMA producer, in both CTAs: its 128 rows of the unit's 256 (the
//             peer skips the copy when the unit ends within the first 128) and
//             its half of B — MODE 0: the leader the 128 gate columns, the peer
//             the 128 up columns; MODE 1: columns 128*rank.. of the 256-column
//             tile. Every copy signals the leader's stage barrier, which the
//             leader arms with the bytes of both CTAs.
//   warp 1    both CTAs allocate and free 512 TMEM columns together (two
//             accumulator buffers of 256). The leader's lane 0 issues
//             tcgen05.mma.cta_group::2, M=256 N=256 K=16: A rows and the D rows
//             split 128 + 128 over the CTAs, B columns 128 + 128. Its commits
//             free the stage and mark the accumulator full in both CTAs.
//   warps 2-5 epilogue in both CTAs, on the CTA's own TMEM (its 128 rows, the
//             M=128 lane layout); releases the accumulator on the leader's
//             barrier.
// Units (expert, 256-row tile, n-tile) are claimed by the leader's producer
// from the atomic counter and published in both CTAs' unit rings (the peer's by
// a remote store and a remote arrive); the peer's readers free ring slots on
// the leader's barrier. Every wait is bounded; a wait that gives up raises
// MOE_DEVERR_TIMEOUT and the roles wind down, and both CTAs still meet at the
// final cluster barrier, so neither leaves while the other may use its shared
// memory or TMEM. All copies fill only the issuing CTA's shared memory.
#include <algorithm>

#include "gemm_tc.cuh"

namespace moe {

namespace tc {

template <int MODE>
struct PairCfg {
    static constexpr int kEpiWarps = 4;
    static constexpr int kThreads = 32 * (2 + kEpiWarps);
    static constexpr int kHalfB = 2 * B_CHUNK;            // 128 N x 64 K: 16 KB
    static constexpr int kStageBytes = A_BYTES + kHalfB;  // 32 KB per CTA
    static constexpr int kStages = 6;
    static constexpr int kSmem = 1024 + kStages * kStageBytes + 512;  // + barriers, unit ring
    static constexpr int kLeaderReaders = 1 + kEpiWarps;  // of the unit ring: MMA, epilogue
    static constexpr int kPeerReaders = 1 + kEpiWarps;    // producer, epilogue
    // M = 256 over the pair; bf16 x bf16 for gate/up, fp16 x fp16 for down; B N-major.
    static constexpr uint32_t kIdesc = idesc_f16_f32(2 * BM, BN, MODE == 0 ? 1 : 0, /*a_mn=*/0, /*b_mn=*/1);
};

// Leader's producer: claim the next unit and publish it in both CTAs' rings.
// The slot is reused once the readers of both CTAs released it. Warp-uniform.
MOE_DEV bool ring_publish_pair(int& u, int& slot, uint32_t& phase, int* counter, int total, volatile int* ring,
                               uint64_t* ufull, uint64_t* uempty, uint32_t peer_ring, uint32_t peer_ufull,
                               volatile int* abort_flag, uint32_t* err, uint64_t ns) {
    const int lane = threadIdx.x & 31;
    int ok = 1;
    if (lane == 0) ok = mbar_wait_bounded<true>(uempty + slot, phase ^ 1u, abort_flag, err, ns);
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    if (!ok) return false;
    int v = 0;
    if (lane == 0) {
        v = atomicAdd(counter, 1);
        if (v >= total) v = -1;
        ring[slot] = v;
        st_shared_cluster_u32(peer_ring + 4u * slot, uint32_t(v));
        mbar_arrive_cluster(peer_ufull + 8u * slot);  // releases the store above
        mbar_arrive(ufull + slot);
    }
    u = __shfl_sync(0xFFFFFFFFu, v, 0);
    if (++slot == UR) {
        slot = 0;
        phase ^= 1u;
    }
    return true;
}

// Peer's readers: the next unit the leader published; the slot is released on
// the leader's barrier. Warp-uniform.
MOE_DEV bool ring_read_peer(int& u, int& slot, uint32_t& phase, volatile int* ring, uint64_t* ufull,
                            uint32_t lead_uempty, volatile int* abort_flag, uint32_t* err, uint64_t ns) {
    const int lane = threadIdx.x & 31;
    int ok = 1;
    if (lane == 0) ok = mbar_wait_bounded<true>(ufull + slot, phase, abort_flag, err, ns);
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    if (!ok) return false;
    int v = 0;
    if (lane == 0) {
        v = ring[slot];
        mbar_arrive_cluster(lead_uempty + 8u * slot);
    }
    u = __shfl_sync(0xFFFFFFFFu, v, 0);
    if (++slot == UR) {
        slot = 0;
        phase ^= 1u;
    }
    return true;
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<MODE>::kThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                             const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmS0,
                             const __grid_constant__ CUtensorMap tmS1, const GemmParams p) {
    using C = PairCfg<MODE>;
    constexpr int STAGES = C::kStages, SB = C::kStageBytes;
    extern __shared__ uint8_t smem_raw[];
    // Every buffer and barrier sits at the same offset in both CTAs: the MMA
    // descriptors and the two-CTA commits address the peer's copy by offset.
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * SB);  // leader: both CTAs' copies landed
    uint64_t* empty = full + STAGES;                                   // both: stage consumed by the MMAs
    uint64_t* tfull = empty + STAGES;                                  // both: accumulator ready
    uint64_t* tempty = tfull + 2;                                      // leader: both epilogues done
    uint64_t* drain = tempty + 2;
    uint64_t* ufull = drain + 1;
    uint64_t* uempty = ufull + UR;  // leader: ring slot read in both CTAs
    volatile int* unit_ring = reinterpret_cast<volatile int*>(uempty + UR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(unit_ring) + UR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = int(cluster_ctarank());
    const bool leader = rank == 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, 2 * C::kEpiWarps);
        }
        for (int r = 0; r < UR; ++r) {
            mbar_init(ufull + r, 1);
            mbar_init(uempty + r, C::kLeaderReaders + C::kPeerReaders);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB0);
        tma_prefetch_desc(&tmB1);
        tma_prefetch_desc(&tmS0);
        tma_prefetch_desc(&tmS1);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    griddep_wait();
    griddep_launch();

    const int nt = p.n_tiles;
    const int total_units = __ldg(p.tile_base + p.Etot) * nt;
    const int KB = p.K / BK;
    const uint32_t lead_uempty = mapa_shared(smem_u32(uempty), 0);

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        const uint32_t lead_full = mapa_shared(smem_u32(full), 0);
        const uint32_t peer_ring = mapa_shared(smem_u32(const_cast<int*>(unit_ring)), 1);
        const uint32_t peer_ufull = mapa_shared(smem_u32(ufull), 1);
        int stage = 0;
        uint32_t phase = 0, issued = 0, issued_par = 0;
        bool ok = true;
        int uslot = 0;
        uint32_t uphase = 0;
        while (ok) {
            int u = -1;
            const bool got = leader ? ring_publish_pair(u, uslot, uphase, p.unit_counter, total_units, unit_ring,
                                                        ufull, uempty, peer_ring, peer_ufull, abort_flag, p.err,
                                                        p.wait_ns)
                                    : ring_read_peer(u, uslot, uphase, unit_ring, ufull, lead_uempty, abort_flag,
                                                     p.err, p.wait_ns);
            if (!got) {
                ok = false;
                break;
            }
            if (u < 0) break;
            const Unit U = decode_unit<2>(u, p, nt);
            const bool sh = U.e >= p.E;
            const int z = sh ? 0 : U.e;
            const bool a_peer = U.rows > BM;  // the peer's 128 rows hold rows of the unit
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
                    uint8_t* sb = sa + A_BYTES;
                    const uint32_t fb = lead_full + 8u * stage;
                    if (leader) mbar_arrive_expect_tx(full + stage, 2u * C::kHalfB + (a_peer ? 2u : 1u) * A_BYTES);
                    if (leader || a_peer) tma_load_2d_pair(sa, &tmA, fb, kb * BK, U.row0 + rank * BM);
                    if (MODE == 0) {
                        const CUtensorMap* m = leader ? (sh ? &tmS0 : &tmB0) : (sh ? &tmS1 : &tmB1);
                        tma_load_4d_pair(sb, m, fb, 0, kb * BK, 2 * U.n, z);  // two 64-column chunks
                    } else {
                        tma_load_4d_pair(sb, sh ? &tmS0 : &tmB0, fb, 0, kb * BK, 4 * U.n + 2 * rank, z);
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
        // On abort, the leader lets every stage it armed complete before the
        // CTAs can leave. The peer's copies signal the same barriers, and a
        // peer that gave up first never issues some of them: those stages
        // cannot complete, so all the waits share one time budget (copies that
        // were issued land within microseconds).
        if (!ok && leader && lane == 0) {
            const uint64_t t_end = globaltimer_ns() + kDrainLimitNs;
            for (int s = 0; s < STAGES; ++s) {
                const uint64_t now = globaltimer_ns();
                if ((issued >> s & 1u) && now < t_end)
                    mbar_wait_bounded(full + s, (issued_par >> s) & 1u, nullptr, p.err, t_end - now);
            }
        }
        // The peer cannot see its own copies complete (they signal the leader's
        // barriers); on abort it gives those it issued 100 us to land.
        if (!ok && !leader && lane == 0 && issued) {
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < 100000ull) {
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader)
        if (leader) {
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
                if (lane == 0)
                    okl = mbar_wait_bounded<true>(tempty + acc, acc_phase ^ 1u, abort_flag, p.err, p.wait_ns);
                okl = __shfl_sync(0xFFFFFFFFu, okl, 0);
                if (!okl) break;
                tc_fence_after();
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
                        const uint32_t a0 = smem_u32(smem + stage * SB);
                        const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
                        for (int j = 0; j < BK / 16; ++j) {
                            // A: K-major, 16 elements = 32 bytes inside the swizzle row.
                            // B: N-major, 16 K-rows = 2 KB; the next 64-column chunk B_CHUNK on.
                            umma_f16_pair(d_tmem, sdesc_sw128(a0 + j * 32, 16, 1024),
                                          sdesc_sw128(b0 + j * 2048, B_CHUNK, 1024), C::kIdesc, (kb | j) != 0);
                        }
                        umma_commit_pair_both(empty + stage);
                    }
                    __syncwarp();
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (lane == 0) umma_commit_pair_both(tfull + acc);
                __syncwarp();
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // every MMA issued has completed before either CTA frees TMEM
            if (lane == 0) {
                umma_commit_pair(drain);
                mbar_wait_bounded(drain, 0, nullptr, p.err, kDrainLimitNs);
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        const uint32_t lead_tempty = mapa_shared(smem_u32(tempty), 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        bool range_bad = false;
        int uslot = 0;
        uint32_t uphase = 0;
        while (true) {
            int u = -1;
            const bool got = leader ? ring_read(u, uslot, uphase, unit_ring, ufull, uempty, abort_flag, p.err,
                                                p.wait_ns)
                                    : ring_read_peer(u, uslot, uphase, unit_ring, ufull, lead_uempty, abort_flag,
                                                     p.err, p.wait_ns);
            if (!got || u < 0) break;
            const Unit U = decode_unit<2>(u, p, nt);
            int okl = 1;
            if (lane == 0) okl = mbar_wait_bounded(tfull + acc, acc_phase, abort_flag, p.err, p.wait_ns);
            okl = __shfl_sync(0xFFFFFFFFu, okl, 0);
            if (!okl) break;
            tc_fence_after();
            const int rows = min(BM, U.rows - rank * BM);
            if (rows > 0) {
                const uint32_t tb = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * BN);
                epilogue_tile<MODE>(tb, U.n, int64_t(U.row0) + rank * BM, rows, /*m64=*/false, q, lane, p,
                                    range_bad);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader) mbar_arrive(tempty + acc);
                else mbar_arrive_cluster(lead_tempty + 8u * acc);
            }
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (range_bad) set_error(p.err, MOE_DEVERR_RANGE);
    }
    __syncthreads();
    tc_fence_before();
    cluster_sync_all();  // both CTAs done with TMEM and with each other's barriers
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

// ---------------------------------------------------------------------------- host side

template <int MODE>
cudaError_t launch_gemm_pair(const CUtensorMap& A, const CUtensorMap& B0, const CUtensorMap& B1, const CUtensorMap& S0,
                             const CUtensorMap& S1, const GemmParams& p, bool pdl, cudaStream_t s) {
    using C = PairCfg<MODE>;
    static int configured_dev = -1, grid = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(grouped_gemm_pair_kernel<MODE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess) return e;
        // One cluster per co-resident SM pair (persistent); units are claimed
        // dynamically, so any grid is correct.
        const int pairs = num_sms() / 2;
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(2 * pairs);
        cfg.blockDim = dim3(C::kThreads);
        cfg.dynamicSmemBytes = C::kSmem;
        int nc = 0;
        if (cudaOccupancyMaxActiveClusters(&nc, grouped_gemm_pair_kernel<MODE>, &cfg) != cudaSuccess || nc < 1) {
            (void)cudaGetLastError();
            nc = pairs;
        }
        grid = 2 * std::min(nc, pairs);
        configured_dev = dev;
    }
    GemmParams q = p;
    q.tile_base = p.tile_base + p.Etot + 1;  // 256-row units
    {
        ProfScope prof_(MODE == 0 ? MOE_K_TC_GATEUP : MOE_K_TC_DOWN, s);
        const cudaError_t le = launch_pdl(pdl, grouped_gemm_pair_kernel<MODE>, dim3(grid), dim3(C::kThreads),
                                          C::kSmem, s, A, B0, B1, S0, S1, q);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

template cudaError_t launch_gemm_pair<0>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                         const CUtensorMap&, const CUtensorMap&, const GemmParams&, bool,
                                         cudaStream_t);
template cudaError_t launch_gemm_pair<1>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                         const CUtensorMap&, const CUtensorMap&, const GemmParams&, bool,
                                         cudaStream_t);

}  // namespace tc

}  // namespace moe

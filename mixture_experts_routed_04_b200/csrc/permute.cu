// permute.cu — S2/S3: per-expert histogram, prefix offsets, scatter and the
// capacity drop, with no atomics.
//
// "mini-AGI PR #3", minagi/pool.py requested(): the (token, expert) pairs are
// flattened, sorted by expert and counted (bincount); with a capacity, a keep
// mask over each expert's sorted pairs drops the overflow and the counts are
// clamped. Here the pairs keep token order inside each expert (pair p = t*k+j
// ranks before p' > p), and the first `cap` of an expert are kept.
//
// Three launches over the T*k pairs, which are cut into blocks of 8 warps x
// ROUNDS rounds of 32 pairs (2 rounds up to 64K pairs, so that the counts and the
// scatter of prompt-sized batches spread over more SMs; 8 rounds above, so that the
// scan over the blocks stays short):
//   count   — each warp counts its pairs per expert (__match_any_sync groups
//             equal ids in a round; the group's lowest lane adds the popcount
//             to the warp's own smem row, so no two lanes write one counter),
//             and the block writes its per-expert totals.
//   scan    — one block: per expert an exclusive scan over blocks gives each
//             block its base; counts, kept = min(count, cap), and an exclusive
//             scan over experts gives offsets.
//   scatter — each block rebuilds its warp totals, turns them into warp bases,
//             and ranks every pair: base + earlier peers in its round. Rank <
//             cap → row offsets[e] + rank.
// The rank of a pair is the number of earlier pairs with the same expert, so
// the result is unique and bit-exact. The shared expert, when present, is
// appended as expert E holding tokens 0..T-1.
#include "schedule.cuh"

namespace moe {

namespace {

MOE_DEV uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Fill hist[w][e] with warp w's pair count per expert for block `b`.
template <int ROUNDS>
MOE_DEV void warp_histograms(const int32_t* __restrict__ topk_idx, int64_t pairs, int E, int (*hist)[kMaxE],
                             uint32_t* err) {
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < kPermWarps * kMaxE; i += blockDim.x) (&hist[0][0])[i] = 0;
    __syncthreads();
    const int64_t base = (int64_t(blockIdx.x) * kPermWarps + w) * (32 * ROUNDS);
    // every round's ids first (one memory latency for the warp's 256 pairs)
    int ids[ROUNDS];
#pragma unroll
    for (int it = 0; it < ROUNDS; ++it) {
        const int64_t p = base + it * 32 + lane;
        int e = -1;
        if (p < pairs) {
            e = __ldg(topk_idx + p);
            if (e < 0 || e >= E) {
                set_error(err, MOE_DEVERR_BOUNDS);
                e = -1;
            }
        }
        ids[it] = e;
    }
#pragma unroll
    for (int it = 0; it < ROUNDS; ++it) {
        const int e = ids[it];
        const uint32_t peers = __match_any_sync(0xFFFFFFFFu, e);
        if (e >= 0 && (__ffs(peers) - 1) == lane) hist[w][e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
}

template <int ROUNDS>
__global__ void __launch_bounds__(kPermWarps * 32) perm_count_kernel(const int32_t* __restrict__ topk_idx,
                                                                     int64_t pairs, int E,
                                                                     int32_t* __restrict__ blockcounts,
                                                                     uint32_t* err) {
    __shared__ int hist[kPermWarps][kMaxE];
    griddep_wait();
    griddep_launch();
    warp_histograms<ROUNDS>(topk_idx, pairs, E, hist, err);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int s = 0;
#pragma unroll
        for (int w = 0; w < kPermWarps; ++w) s += hist[w][e];
        blockcounts[int64_t(blockIdx.x) * E + e] = s;
    }
}

// One block: thread e owns expert e (256 threads; 512 with SCHED). With SCHED
// the block then runs the tile schedule on the kept counts it has just formed
// (the schedule kernel's work, without a launch of its own).
template <bool SCHED>
__global__ void __launch_bounds__(SCHED ? 512 : kMaxE)
    perm_scan_kernel(const int32_t* __restrict__ blockcounts, int nblocks, int E, int cap, int shared_T,
                     int32_t* __restrict__ blockbase, int32_t* __restrict__ counts, int32_t* __restrict__ kept,
                     int32_t* __restrict__ offsets, ScheduleArgs sa) {
    __shared__ int warp_sums[16];
    __shared__ int sums[3][16];
    griddep_wait();
    griddep_launch();

    const int e = threadIdx.x, lane = e & 31, w = e >> 5;
    const int nw = blockDim.x >> 5;
    int kv = 0;
    if (e < E) {
        int run = 0;
#pragma unroll 8
        for (int b = 0; b < nblocks; ++b) {
            const int c = blockcounts[int64_t(b) * E + e];
            blockbase[int64_t(b) * E + e] = run;
            run += c;
        }
        counts[e] = run;
        kv = (cap >= 0 && run > cap) ? cap : run;
        kept[e] = kv;
    }
    // exclusive scan of kv over the block
    int incl = kv;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) warp_sums[w] = incl;
    __syncthreads();
    int wbase = 0, total = 0;
    for (int i = 0; i < nw; ++i) {
        if (i < w) wbase += warp_sums[i];
        total += warp_sums[i];
    }
    if (e < E) offsets[e] = wbase + incl - kv;
    if (e == 0) {
        if (shared_T > 0) {
            counts[E] = shared_T;
            kept[E] = shared_T;
            offsets[E] = total;
            offsets[E + 1] = total + shared_T;
        } else {
            offsets[E] = total;
        }
    }
    if (SCHED) {
        const int Etot = E + (shared_T > 0 ? 1 : 0);
        const int ke = e < E ? kv : (e == E && shared_T > 0 ? shared_T : 0);
        schedule_block(ke, Etot, sa.variant, sa.stream_max, sums, sa.tile_base, sa.stream_list, sa.n_stream);
    }
}

// The scan's outputs a fused scatter block forms itself (FUSED; perm_scan_kernel otherwise).
struct ScanOut {
    const int32_t* blockcounts;  // [nblocks][E] from the count pass (16-byte aligned)
    int nblocks;
    int32_t* counts;             // block 0 writes counts, kept, offsets and the schedule
    int32_t* kept;
    int32_t* offsets;
    ScheduleArgs sa;
};

// FUSED: the per-block counts are copied to shared memory (dynamic, nblocks * E
// ints) and every block forms its base (its earlier blocks' counts, per expert)
// and the expert offsets itself, in the scan kernel's order, so no scan launch is
// made; offsets then come from shared memory instead of the scan's output.
template <int ROUNDS, bool FUSED>
__global__ void __launch_bounds__(kPermWarps * 32) perm_scatter_kernel(
    const int32_t* __restrict__ topk_idx, int64_t pairs, int k, int E, int cap,
    const int32_t* __restrict__ blockbase, const int32_t* __restrict__ offsets,
    int32_t* __restrict__ sorted_token, int32_t* __restrict__ sorted_pair, int32_t* __restrict__ pair_row,
    int shared_T, uint32_t* err, ScanOut so) {
    __shared__ int hist[kPermWarps][kMaxE];
    __shared__ int s_base[FUSED ? kMaxE : 1];
    __shared__ int s_off[FUSED ? kMaxE + 1 : 1];
    __shared__ int warp_sums[kPermWarps];
    __shared__ int sums[3][16];
    extern __shared__ int4 s_counts4[];
    griddep_wait();
    griddep_launch();
    if (FUSED) {
        const int* s_counts = reinterpret_cast<const int*>(s_counts4);
        const int n = so.nblocks * E;
        const int n4 = n >> 2;
        const int4* src4 = reinterpret_cast<const int4*>(so.blockcounts);
#pragma unroll 4
        for (int i = threadIdx.x; i < n4; i += blockDim.x) s_counts4[i] = src4[i];
        for (int i = 4 * n4 + threadIdx.x; i < n; i += blockDim.x)
            reinterpret_cast<int*>(s_counts4)[i] = so.blockcounts[i];
        __syncthreads();
        const int e = threadIdx.x, lane = e & 31, w = e >> 5;
        int kv = 0;
        if (e < E) {
            int before = 0, total = 0;
#pragma unroll 8
            for (int b = 0; b < so.nblocks; ++b) {
                const int c = s_counts[b * E + e];
                total += c;
                before += b < int(blockIdx.x) ? c : 0;
            }
            s_base[e] = before;
            kv = (cap >= 0 && total > cap) ? cap : total;
            if (blockIdx.x == 0) {
                so.counts[e] = total;
                so.kept[e] = kv;
            }
        }
        // exclusive scan of kv over the experts
        int incl = kv;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off) incl += v;
        }
        if (lane == 31) warp_sums[w] = incl;
        __syncthreads();
        int wbase = 0, routed = 0;
#pragma unroll
        for (int i = 0; i < kPermWarps; ++i) {
            if (i < w) wbase += warp_sums[i];
            routed += warp_sums[i];
        }
        if (e < E) s_off[e] = wbase + incl - kv;
        if (e == 0) s_off[E] = routed;
        if (blockIdx.x == 0) {
            if (e < E) so.offsets[e] = wbase + incl - kv;
            if (e == 0) {
                so.offsets[E] = routed;
                if (shared_T > 0) {
                    so.counts[E] = shared_T;
                    so.kept[E] = shared_T;
                    so.offsets[E + 1] = routed + shared_T;
                }
            }
            const int Etot = E + (shared_T > 0 ? 1 : 0);
            const int ke = e < E ? kv : (e == E && shared_T > 0 ? shared_T : 0);
            schedule_block(ke, Etot, so.sa.variant, so.sa.stream_max, sums, so.sa.tile_base, so.sa.stream_list,
                           so.sa.n_stream);
        }
        __syncthreads();
    }
    warp_histograms<ROUNDS>(topk_idx, pairs, E, hist, nullptr);  // errors were reported by the count pass
    // warp totals -> warp bases (block base + earlier warps), per expert
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = FUSED ? s_base[e] : blockbase[int64_t(blockIdx.x) * E + e];
#pragma unroll
        for (int w = 0; w < kPermWarps; ++w) {
            const int c = hist[w][e];
            hist[w][e] = run;
            run += c;
        }
    }
    __syncthreads();
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t base = (int64_t(blockIdx.x) * kPermWarps + w) * (32 * ROUNDS);
    int ids[ROUNDS];
#pragma unroll
    for (int it = 0; it < ROUNDS; ++it) {
        const int64_t p = base + it * 32 + lane;
        int e = -1;
        if (p < pairs) {
            e = __ldg(topk_idx + p);
            if (e < 0 || e >= E) e = -1;
        }
        ids[it] = e;
    }
#pragma unroll
    for (int it = 0; it < ROUNDS; ++it) {
        const int64_t p = base + it * 32 + lane;
        const int e = ids[it];
        const uint32_t peers = __match_any_sync(0xFFFFFFFFu, e);
        int rank = 0;
        if (e >= 0) rank = hist[w][e] + __popc(peers & lanemask_lt());
        __syncwarp();
        if (e >= 0 && (__ffs(peers) - 1) == lane) hist[w][e] += __popc(peers);
        __syncwarp();
        if (p < pairs) {
            if (e >= 0 && (cap < 0 || rank < cap)) {
                const int row = (FUSED ? s_off[e] : offsets[e]) + rank;
                sorted_token[row] = int32_t(p / k);
                sorted_pair[row] = int32_t(p);
                pair_row[p] = row;
            } else {
                pair_row[p] = -1;
            }
        }
    }
    // shared-expert rows: tokens 0..T-1 after the routed rows
    if (shared_T > 0) {
        const int base_row = FUSED ? s_off[E] : offsets[E];
        for (int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; t < shared_T;
             t += int64_t(gridDim.x) * blockDim.x) {
            sorted_token[base_row + t] = int32_t(t);
            sorted_pair[base_row + t] = -1;
        }
    }
}

}  // namespace

cudaError_t launch_permute(const Dims& D, const int32_t* topk_idx, int32_t* blockcounts, int32_t* blockbase,
                           int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* sorted_token,
                           int32_t* sorted_pair, int32_t* pair_row, uint32_t* err, cudaStream_t s,
                           const ScheduleArgs* sched) {
    if (D.pairs == 0) {  // empty batch: zero counts and offsets, nothing to scatter
        if (cudaMemsetAsync(counts, 0, size_t(D.Etot) * 4, s) != cudaSuccess ||
            cudaMemsetAsync(kept, 0, size_t(D.Etot) * 4, s) != cudaSuccess ||
            cudaMemsetAsync(offsets, 0, size_t(D.Etot + 1) * 4, s) != cudaSuccess)
            return cudaGetLastError();
        return cudaSuccess;
    }
    const int nb = D.perm_blocks;
    const int shared_T = D.has_shared ? D.T : 0;
    {
        ProfScope prof_(MOE_K_PERM_COUNT, s);
        const bool small = perm_rounds(D.pairs) == kPermRoundsSmall;
        const cudaError_t le =
            small ? launch_pdl(use_pdl(D.T), perm_count_kernel<kPermRoundsSmall>, dim3(nb), dim3(kPermWarps * 32), 0,
                               s, topk_idx, D.pairs, D.E, blockcounts, err)
                  : launch_pdl(use_pdl(D.T), perm_count_kernel<kPermRoundsLarge>, dim3(nb), dim3(kPermWarps * 32), 0,
                               s, topk_idx, D.pairs, D.E, blockcounts, err);
        if (le != cudaSuccess) return le;
    }
    const bool fused = sched && perm_scan_fused(D);
    if (!fused) {
        ProfScope prof_(MOE_K_PERM_SCAN, s);
        const ScheduleArgs none{};
        const cudaError_t le =
            sched ? launch_pdl(use_pdl(D.T), perm_scan_kernel<true>, dim3(1), dim3(512), 0, s, blockcounts, nb, D.E,
                               D.cap, shared_T, blockbase, counts, kept, offsets, *sched)
                  : launch_pdl(use_pdl(D.T), perm_scan_kernel<false>, dim3(1), dim3(kMaxE), 0, s, blockcounts, nb,
                               D.E, D.cap, shared_T, blockbase, counts, kept, offsets, none);
        if (le != cudaSuccess) return le;
    }
    {
        ProfScope prof_(MOE_K_PERM_SCATTER, s);
        const bool small = perm_rounds(D.pairs) == kPermRoundsSmall;
        cudaError_t le;
        if (fused) {
            static int configured_dev = -1;
            int dev = 0;
            cudaGetDevice(&dev);
            if (configured_dev != dev) {
                if ((le = cudaFuncSetAttribute(perm_scatter_kernel<kPermRoundsSmall, true>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, kScanFusedMaxBytes)) !=
                        cudaSuccess ||
                    (le = cudaFuncSetAttribute(perm_scatter_kernel<kPermRoundsLarge, true>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, kScanFusedMaxBytes)) !=
                        cudaSuccess)
                    return le;
                configured_dev = dev;
            }
            const ScanOut so{blockcounts, nb, counts, kept, offsets, *sched};
            const int smem = nb * D.E * 4;
            le = small ? launch_pdl(use_pdl(D.T), perm_scatter_kernel<kPermRoundsSmall, true>, dim3(nb),
                                    dim3(kPermWarps * 32), smem, s, topk_idx, D.pairs, D.k, D.E, D.cap, blockbase,
                                    offsets, sorted_token, sorted_pair, pair_row, shared_T, err, so)
                       : launch_pdl(use_pdl(D.T), perm_scatter_kernel<kPermRoundsLarge, true>, dim3(nb),
                                    dim3(kPermWarps * 32), smem, s, topk_idx, D.pairs, D.k, D.E, D.cap, blockbase,
                                    offsets, sorted_token, sorted_pair, pair_row, shared_T, err, so);
        } else {
            const ScanOut none{};
            le = small ? launch_pdl(use_pdl(D.T), perm_scatter_kernel<kPermRoundsSmall, false>, dim3(nb),
                                    dim3(kPermWarps * 32), 0, s, topk_idx, D.pairs, D.k, D.E, D.cap, blockbase,
                                    offsets, sorted_token, sorted_pair, pair_row, shared_T, err, none)
                       : launch_pdl(use_pdl(D.T), perm_scatter_kernel<kPermRoundsLarge, false>, dim3(nb),
                                    dim3(kPermWarps * 32), 0, s, topk_idx, D.pairs, D.k, D.E, D.cap, blockbase,
                                    offsets, sorted_token, sorted_pair, pair_row, shared_T, err, none);
        }
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe

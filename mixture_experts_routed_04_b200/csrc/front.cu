// front.cu — S1..S3 and K3 for small batches in one block: routing, counts,
// capacity, offsets, the token-order scatter and the tile schedule, for at
// most kFrontMaxTokens tokens (T*k <= 512 pairs, one pair per thread), and for
// the smallest batches (at most kFrontGatherBytes of rows) the S4 row gather
// too. At a few tokens the separate kernels are each a launch and a few
// dependent memory round trips; here they are one. The results are those of
// the separate kernels: the routing and the schedule run the same device code,
// and the ranks (earlier pairs of the same expert, in token order) are unique.
#include "route.cuh"
#include "schedule.cuh"

namespace moe {

namespace {

constexpr int kFrontThreads = 512;
constexpr int kFrontWarps = kFrontThreads / 32;

MOE_DEV uint32_t lanemask_lt_front() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__global__ void __launch_bounds__(kFrontThreads)
    front_small_kernel(const float* __restrict__ logits, int T, int E, int k, int cap, int has_shared, int variant,
                       int stream_max, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                       int32_t* __restrict__ counts, int32_t* __restrict__ kept_out, int32_t* __restrict__ offsets,
                       int32_t* __restrict__ sorted_token, int32_t* __restrict__ sorted_pair,
                       int32_t* __restrict__ pair_row, int32_t* __restrict__ tile_base,
                       int32_t* __restrict__ stream_list, int32_t* __restrict__ n_stream,
                       const uint16_t* __restrict__ x, int d, uint16_t* __restrict__ xg,
                       int32_t* __restrict__ comb_count, int ncomb, uint32_t* err) {
    __shared__ int hist[kFrontWarps][kMaxE];  // per-warp counts per expert, then warp bases
    __shared__ int s_off[kMaxE + 2];
    __shared__ int s_tok[kFrontThreads + kFrontMaxTokens];  // token of each row (S4, when gathering)
    __shared__ int wsum[kFrontWarps];
    __shared__ int sums[3][16];
    griddep_wait();
    griddep_launch();
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int pairs = T * k;
    if (comb_count)
        for (int i = tid; i < ncomb; i += kFrontThreads) comb_count[i] = 0;

    // S1: warp w routes tokens w, w + 16, ...
    for (int t = w; t < T; t += kFrontWarps)
        route_one_token(logits + int64_t(t) * E, E, k, topk_idx + int64_t(t) * k, topk_w + int64_t(t) * k);
    for (int i = tid; i < kFrontWarps * kMaxE; i += kFrontThreads) (&hist[0][0])[i] = 0;
    __syncthreads();  // the block's topk_idx writes are visible to the block

    // S2: pair p = tid; the warp's peers with the same expert, counted once per group
    int e = -1;
    if (tid < pairs) {
        e = topk_idx[tid];
        if (e < 0 || e >= E) {
            set_error(err, MOE_DEVERR_BOUNDS);
            e = -1;
        }
    }
    const uint32_t peers = __match_any_sync(0xFFFFFFFFu, e);
    if (e >= 0 && (__ffs(peers) - 1) == lane) hist[w][e] = __popc(peers);
    __syncthreads();
    // thread x owns expert x: count, warp bases, kept (the shared expert is index E, T rows)
    const int Etot = E + has_shared;
    int kv = 0;
    if (tid < E) {
        int run = 0;
#pragma unroll
        for (int i = 0; i < kFrontWarps; ++i) {
            const int c = hist[i][tid];
            hist[i][tid] = run;
            run += c;
        }
        counts[tid] = run;
        kv = (cap >= 0 && run > cap) ? cap : run;
        kept_out[tid] = kv;
    } else if (tid == E && has_shared) {
        counts[E] = T;
        kept_out[E] = T;
        kv = T;
    }
    // offsets: exclusive scan of kept over the experts (routed, then the shared one)
    int incl = kv;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) wsum[w] = incl;
    __syncthreads();
    int wbase = 0, total = 0;
#pragma unroll
    for (int i = 0; i < kFrontWarps; ++i) {
        if (i < w) wbase += wsum[i];
        total += wsum[i];
    }
    if (tid < Etot) {
        offsets[tid] = wbase + incl - kv;
        s_off[tid] = wbase + incl - kv;
    }
    if (tid == 0) offsets[Etot] = total;
    __syncthreads();

    // S3: rank = earlier pairs of the same expert; rank < cap keeps the pair
    if (tid < pairs) {
        int row = -1;
        if (e >= 0) {
            const int rank = hist[w][e] + __popc(peers & lanemask_lt_front());
            if (cap < 0 || rank < cap) {
                row = s_off[e] + rank;
                sorted_token[row] = tid / k;
                sorted_pair[row] = tid;
                s_tok[row] = tid / k;
            }
        }
        pair_row[tid] = row;
    }
    if (has_shared)
        for (int t = tid; t < T; t += kFrontThreads) {
            sorted_token[s_off[E] + t] = t;
            sorted_pair[s_off[E] + t] = -1;
            s_tok[s_off[E] + t] = t;
        }

    // S4 (smallest batches): xg[r] = x[token of r], 16-byte vectors, four loads in flight a thread
    if (xg) {
        __syncthreads();
        const int vec = d / 8;
        const int64_t nvec = int64_t(total) * vec;
        for (int64_t i0 = tid; i0 < nvec; i0 += 4 * kFrontThreads) {
            uint4 v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t i = i0 + int64_t(j) * kFrontThreads;
                if (i < nvec) {
                    const int r = int(i / vec), c = int(i - int64_t(r) * vec);
                    v[j] = __ldg(reinterpret_cast<const uint4*>(x + int64_t(s_tok[r]) * d) + c);
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t i = i0 + int64_t(j) * kFrontThreads;
                if (i < nvec) reinterpret_cast<uint4*>(xg)[i] = v[j];
            }
        }
    }

    // K3: the tile schedule from the kept counts (thread x owns expert x)
    schedule_block(tid < Etot ? kv : 0, Etot, variant, stream_max, sums, tile_base, stream_list, n_stream);
}

}  // namespace

// Rows can number at most T*k + T (every pair kept, plus the shared expert's).
bool front_gathers(const Dims& D) {
    const int64_t rows = int64_t(D.T) * D.k + (D.has_shared ? D.T : 0);
    return D.fmt == MOE_WEIGHTS_BF16 && D.T <= kFrontMaxTokens && rows * D.d * 2 <= kFrontGatherBytes;
}

cudaError_t launch_front_small(const Dims& D, const float* logits, int32_t* topk_idx, float* topk_w,
                               int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* sorted_token,
                               int32_t* sorted_pair, int32_t* pair_row, int32_t* tile_base, int32_t* stream_list,
                               int32_t* n_stream, const uint16_t* x, uint16_t* xg, int32_t* comb_count,
                               uint32_t* err, cudaStream_t s) {
    if (D.T > kFrontMaxTokens || int64_t(D.T) * D.k > kFrontThreads || D.E > kMaxE) return cudaErrorInvalidValue;
    if (xg && (!x || !front_gathers(D))) return cudaErrorInvalidValue;
    {
        ProfScope prof_(MOE_K_FRONT, s);
        const cudaError_t le = launch_pdl(use_pdl(D.T), front_small_kernel, dim3(1), dim3(kFrontThreads), 0, s,
                                          logits, D.T, D.E, D.k, D.cap, D.has_shared, D.variant, D.stream_max_rows,
                                          topk_idx, topk_w, counts, kept, offsets, sorted_token, sorted_pair,
                                          pair_row, tile_base, stream_list, n_stream, x, D.d, xg, comb_count,
                                          combine_blocks(D), err);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe

// route.cu — S1: top-k routing with a softmax over the selected logits.
//
// "mini-AGI PR #3", minagi/pool.py requested(): probs = softmax(logits), the
// top-k of probs, renormalised. Renormalising the top-k of a full softmax is a
// softmax over the k selected logits; that is what is computed, in fp32.
//
// One warp per token (route_one_token in route.cuh). Each lane keeps up to 8 of
// the E <= 256 logits as order-preserving integer keys (expert lane + 32*i).
// k rounds pick the experts in descending order: every lane offers its best
// untaken key, one warp max-reduction gives the winning value and one
// min-reduction over the lanes holding it the lowest expert index, so equal
// values go to the lower index and -0.0 equals +0.0 (the keys are built from
// the given values, never from recomputed probabilities): the indices are
// bit-exact.
#include "route.cuh"

namespace moe {

namespace {

// One warp per token (route_one_token, shared with the fused small-batch front kernel).
__global__ void __launch_bounds__(256) route_topk_softmax_kernel(const float* __restrict__ logits, int T, int E,
                                                                 int k, int32_t* __restrict__ topk_idx,
                                                                 float* __restrict__ topk_w) {
    griddep_wait();
    griddep_launch();
    const int warps_per_block = blockDim.x >> 5;
    const int64_t t = int64_t(blockIdx.x) * warps_per_block + (threadIdx.x >> 5);
    if (t >= T) return;
    route_one_token(logits + t * E, E, k, topk_idx + t * k, topk_w + t * k);
}


// ---------------------------------------------------------------- router telemetry
//
// "mini-AGI PR #3", requested(), telemetry hunk, on the full softmax p of
// each token's logits: kept = the top-k mass before renormalisation; want =
// the fewest experts (largest first) whose mass reaches 90%; balance =
// E * sum_e frac_e * mean_t p[t, e] (frac_e: share of tokens whose first
// choice is e); z = mean_t logsumexp(logits[t])^2; aux = balance + z_w * z.
//
// route_stats_kernel: one warp per token as in the router (the same
// route_one_token, so idx and w are those of moe_route), then over the same
// token: max and sum of exp over all E (warp reductions), and selection
// rounds in descending order (ties to the lower index) summing exp in that
// order until the top-k mass and the 90% count are both known. Each block
// keeps per-expert sums of p and first-choice counts, reduced over its warps
// in warp order into one row of partials; route_stats_final sums the rows in
// block order (fp64). Fixed orders throughout: the results are deterministic.

constexpr int kStatsWarps = 8;
constexpr float kWantMass = 0.9f;

template <bool PER_TOKEN>
__global__ void __launch_bounds__(kStatsWarps * 32)
    route_stats_kernel(const float* __restrict__ logits, int T, int E, int k, int32_t* __restrict__ topk_idx,
                       float* __restrict__ topk_w, float* __restrict__ kept_tok, int32_t* __restrict__ want_tok,
                       float* __restrict__ part_p, int32_t* __restrict__ part_c, float* __restrict__ part_s) {
    __shared__ float sp[kStatsWarps][kMaxE];
    __shared__ int sc[kStatsWarps][kMaxE];
    __shared__ float ss[kStatsWarps][3];
    griddep_wait();
    griddep_launch();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    float accp[kRouteMaxPerLane];
    int accc[kRouteMaxPerLane];
#pragma unroll
    for (int i = 0; i < kRouteMaxPerLane; ++i) {
        accp[i] = 0.f;
        accc[i] = 0;
    }
    float a_kept = 0.f, a_want = 0.f, a_z = 0.f;
    for (int64_t t = int64_t(blockIdx.x) * kStatsWarps + w; t < T; t += int64_t(gridDim.x) * kStatsWarps) {
        const float* row = logits + t * E;
        const int first = route_one_token(row, E, k, topk_idx + t * k, topk_w + t * k);
        float v[kRouteMaxPerLane];
        uint32_t key[kRouteMaxPerLane];
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < kRouteMaxPerLane; ++i) {
            const int e = lane + 32 * i;
            v[i] = e < E ? __ldg(row + e) : -INFINITY;
            key[i] = e < E ? route_key(v[i]) : 0u;
            mx = fmaxf(mx, v[i]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
        float ex[kRouteMaxPerLane], S = 0.f;
#pragma unroll
        for (int i = 0; i < kRouteMaxPerLane; ++i) {
            ex[i] = lane + 32 * i < E ? expf(v[i] - mx) : 0.f;
            S += ex[i];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) S += __shfl_xor_sync(0xFFFFFFFFu, S, off);
        const float inv = 1.0f / S;
#pragma unroll
        for (int i = 0; i < kRouteMaxPerLane; ++i) {
            accp[i] += ex[i] * inv;
            accc[i] += (lane + 32 * i == first) ? 1 : 0;
        }
        // selection rounds, largest first, ties to the lower index (as the router)
        uint32_t taken = 0;
#pragma unroll
        for (int i = 0; i < kRouteMaxPerLane; ++i)
            if (lane + 32 * i >= E) taken |= 1u << i;
        const float thr = kWantMass * S;
        float cum = 0.f, kept_t = 0.f;
        int want = 0;
        for (int r = 0; r < E; ++r) {
            uint32_t bk = 0;
            int bi = 0x7FFFFFFF;
#pragma unroll
            for (int i = 0; i < kRouteMaxPerLane; ++i)
                if (!(taken >> i & 1u) && (key[i] > bk || bi == 0x7FFFFFFF)) {
                    bk = key[i];
                    bi = lane + 32 * i;
                }
            const uint32_t kmax = __reduce_max_sync(0xFFFFFFFFu, bk);
            const int wi =
                int(__reduce_min_sync(0xFFFFFFFFu, (bi != 0x7FFFFFFF && bk == kmax) ? uint32_t(bi) : 0xFFFFFFFFu));
            if ((wi & 31) == lane) taken |= 1u << (wi >> 5);
            cum += expf(route_unkey(kmax) - mx);
            if (r == k - 1) kept_t = cum * inv;
            if (want == 0 && cum >= thr) want = r + 1;
            if (want != 0 && r >= k - 1) break;
        }
        if (want == 0) want = E;  // the whole mass, up to rounding
        a_kept += kept_t;
        a_want += float(want);
        const float lse = mx + logf(S);
        a_z += lse * lse;
        if (PER_TOKEN && lane == 0) {
            if (kept_tok) kept_tok[t] = kept_t;
            if (want_tok) want_tok[t] = want;
        }
    }
#pragma unroll
    for (int i = 0; i < kRouteMaxPerLane; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            sp[w][e] = accp[i];
            sc[w][e] = accc[i];
        }
    }
    if (lane == 0) {
        ss[w][0] = a_kept;
        ss[w][1] = a_want;
        ss[w][2] = a_z;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float a = 0.f;
        int c = 0;
        for (int j = 0; j < kStatsWarps; ++j) {
            a += sp[j][e];
            c += sc[j][e];
        }
        part_p[int64_t(blockIdx.x) * E + e] = a;
        part_c[int64_t(blockIdx.x) * E + e] = c;
    }
    if (threadIdx.x < 3) {
        float a = 0.f;
        for (int j = 0; j < kStatsWarps; ++j) a += ss[j][threadIdx.x];
        part_s[blockIdx.x * 3 + threadIdx.x] = a;
    }
}

// One block: thread e sums expert e's partial rows in block order; then the
// scalars. stats = {kept, want_k, balance, z, aux}; expert_stats (nullable) =
// {frac [E], prob_mean [E]}.
__global__ void __launch_bounds__(kMaxE) route_stats_final(const float* __restrict__ part_p,
                                                          const int32_t* __restrict__ part_c,
                                                          const float* __restrict__ part_s, int nblk, int T, int E,
                                                          float z_weight, float* __restrict__ stats,
                                                          float* __restrict__ expert_stats) {
    __shared__ double term[kMaxE];
    griddep_wait();
    griddep_launch();
    const int e = threadIdx.x;
    double pm = 0.0;
    long long cnt = 0;
    if (e < E) {
        for (int b = 0; b < nblk; ++b) {
            pm += double(part_p[int64_t(b) * E + e]);
            cnt += part_c[int64_t(b) * E + e];
        }
        pm /= double(T);
        const double frac = double(cnt) / double(T);
        term[e] = frac * pm;
        if (expert_stats) {
            expert_stats[e] = float(frac);
            expert_stats[E + e] = float(pm);
        }
    }
    __syncthreads();
    if (e == 0) {
        double bal = 0.0, s[3] = {0.0, 0.0, 0.0};
        for (int j = 0; j < E; ++j) bal += term[j];
        bal *= double(E);
        for (int b = 0; b < nblk; ++b)
            for (int j = 0; j < 3; ++j) s[j] += double(part_s[b * 3 + j]);
        const double z = s[2] / double(T);
        stats[0] = float(s[0] / double(T));
        stats[1] = float(s[1] / double(T));
        stats[2] = float(bal);
        stats[3] = float(z);
        stats[4] = float(bal + double(z_weight) * z);
    }
}

}  // namespace

// Blocks of the telemetry kernel: enough tokens per block to keep its partial
// rows few (the final sum is one block), enough blocks to fill the GPU.
int route_stats_blocks(int T) {
    const int need = (T + kStatsWarps - 1) / kStatsWarps;
    return need < 2 * num_sms() ? need : 2 * num_sms();
}

cudaError_t launch_route_stats(const float* logits, int T, int E, int k, int32_t* topk_idx, float* topk_w,
                               float z_weight, float* stats, float* kept_tok, int32_t* want_tok,
                               float* expert_stats, float* part_p, int32_t* part_c, float* part_s,
                               cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    const int nb = route_stats_blocks(T);
    const bool pdl = use_pdl(T);
    {
        ProfScope prof_(MOE_K_ROUTE, stream);
        const cudaError_t le =
            (kept_tok || want_tok)
                ? launch_pdl(pdl, route_stats_kernel<true>, dim3(nb), dim3(kStatsWarps * 32), 0, stream, logits, T,
                             E, k, topk_idx, topk_w, kept_tok, want_tok, part_p, part_c, part_s)
                : launch_pdl(pdl, route_stats_kernel<false>, dim3(nb), dim3(kStatsWarps * 32), 0, stream, logits,
                             T, E, k, topk_idx, topk_w, kept_tok, want_tok, part_p, part_c, part_s);
        if (le != cudaSuccess) return le;
    }
    {
        ProfScope prof_(MOE_K_ROUTE_STATS, stream);
        const cudaError_t le = launch_pdl(pdl, route_stats_final, dim3(1), dim3(kMaxE), 0, stream, part_p, part_c,
                                          part_s, nb, T, E, z_weight, stats, expert_stats);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* topk_idx, float* topk_w,
                         cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    const int threads = 256, wpb = threads / 32;
    const int blocks = (T + wpb - 1) / wpb;
    {
        ProfScope prof_(MOE_K_ROUTE, stream);
        const cudaError_t le = launch_pdl(use_pdl(T), route_topk_softmax_kernel, dim3(blocks), dim3(threads), 0,
                                          stream, logits, T, E, k, topk_idx, topk_w);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe

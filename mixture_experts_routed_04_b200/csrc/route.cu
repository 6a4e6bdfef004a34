// route.cu — S1: top-k routing with a softmax over the selected logits.
//
// "mini-AGI PR #3", minagi/pool.py requested(): probs = softmax(logits), the
// top-k of probs, renormalised. Renormalising the top-k of a full softmax is a
// softmax over the k selected logits; that is what is computed, in fp32.
//
// One warp per token (route_one_token in route.cuh). Each lane keeps up to 8 of
// the E <= 256 logits (4 in this kernel when E <= 128) as order-preserving integer
// keys (expert lane + 32*i).
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
    if (E <= 128)  // four keys a lane: half the selection work of the 256-expert form
        route_one_token<4>(logits + t * E, E, k, topk_idx + t * k, topk_w + t * k);
    else
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
// token: max and sum of exp over all E (warp reductions); the top-k mass from
// the k-th selected key (every value above it plus enough of its ties); the
// 90% count by bisection over the 32-bit order-preserving keys for the
// largest threshold whose values hold >= 90% of the mass (32 rounds of a masked
// warp sum, whatever E), then as many of that value's ties as the remaining
// mass needs — the count of the largest-first definition. Each block
// keeps per-expert sums of p and first-choice counts, reduced over its warps
// in warp order into one row of partials; route_stats_final sums the rows
// (fp64, lanes over block rows, then a fixed shuffle tree). Fixed orders
// throughout: the results are deterministic.

constexpr int kStatsWarps = 16;
// Partial rows a lane of the final sum reads: the telemetry kernel runs at most
// 32 x this many blocks (route_stats_blocks).
constexpr int kStatsMaxRowsPerLane = 8;
constexpr float kWantMass = 0.9f;

template <bool PER_TOKEN>
__global__ void __launch_bounds__(kStatsWarps * 32, 2)
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
        uint32_t kth = 0;
        const int first = route_one_token(row, E, k, topk_idx + t * k, topk_w + t * k, &kth);
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
        // mass and count of the values whose key is > tau (over the valid experts)
        auto above = [&](uint32_t tau, float& mass, int& cnt) {
            float m = 0.f;
            int c = 0;
#pragma unroll
            for (int i = 0; i < kRouteMaxPerLane; ++i)
                if (lane + 32 * i < E && key[i] > tau) {
                    m += ex[i];
                    ++c;
                }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                m += __shfl_xor_sync(0xFFFFFFFFu, m, off);
                c += __shfl_xor_sync(0xFFFFFFFFu, c, off);
            }
            mass = m;
            cnt = c;
        };
        // kept: the k selected = every value above the k-th key plus enough of its ties
        float m_above;
        int c_above;
        above(kth, m_above, c_above);
        const float e_kth = expf(route_unkey(kth) - mx);
        const float kept_t = (m_above + float(k - c_above) * e_kth) * inv;
        // want: tau* = the largest key whose values at or above it hold >= 90% of the mass
        // (bisection over the 32-bit keys; mass(key >= tau) = mass(key > tau - 1)); then
        // the values above tau* plus as many of its ties as the remaining mass needs, in
        // the largest-first order of the definition
        const float thr = kWantMass * S;
        // the rounds need only the mass (one warp sum; the count is taken once at the end)
        auto mass_above = [&](uint32_t tau) {
            float m = 0.f;
#pragma unroll
            for (int i = 0; i < kRouteMaxPerLane; ++i)
                if (lane + 32 * i < E && key[i] > tau) m += ex[i];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m += __shfl_xor_sync(0xFFFFFFFFu, m, off);
            return m;
        };
        uint32_t lo = 0u, hi = 0xFFFFFFFFu;
        while (lo < hi) {
            const uint32_t mid = lo + ((hi - lo) >> 1) + 1u;
            if (mass_above(mid - 1u) >= thr) lo = mid;
            else hi = mid - 1u;
        }
        above(lo, m_above, c_above);
        const float e_tau = expf(route_unkey(lo) - mx);
        int want = c_above;
        float cum = m_above;
        do {
            cum += e_tau;
            ++want;
        } while (cum < thr && want < E);
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
        // expert-major [E, blocks]: the final sum reads each expert's rows contiguously
        part_p[int64_t(e) * gridDim.x + blockIdx.x] = a;
        part_c[int64_t(e) * gridDim.x + blockIdx.x] = c;
    }
    if (threadIdx.x < 3) {
        float a = 0.f;
        for (int j = 0; j < kStatsWarps; ++j) a += ss[j][threadIdx.x];
        part_s[blockIdx.x * 3 + threadIdx.x] = a;
    }
}

// One block of 1024 threads: warp w takes experts w, w + 32, ...; lane l sums
// block rows l, l + 32, ... (fp64; the partials are expert-major, so a warp's
// loads are coalesced) and a fixed shuffle tree adds the lanes, so
// the order of every sum is fixed. Then warp 0 sums the balance terms and the
// scalars the same way. stats = {kept, want_k, balance, z, aux}; expert_stats
// (nullable) = {frac [E], prob_mean [E]}.
MOE_DEV double warp_sum_fixed(double v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
    return v;
}

__global__ void __launch_bounds__(1024) route_stats_final(const float* __restrict__ part_p,
                                                          const int32_t* __restrict__ part_c,
                                                          const float* __restrict__ part_s, int nblk, int T, int E,
                                                          float z_weight, float* __restrict__ stats,
                                                          float* __restrict__ expert_stats) {
    __shared__ double term[kMaxE];
    griddep_wait();
    griddep_launch();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int e = w; e < E; e += 32) {
        // this lane's block rows b = lane + 32 j, loaded into registers first (all in
        // flight together), then summed in j order
        float vp[kStatsMaxRowsPerLane];
        int vc[kStatsMaxRowsPerLane];
#pragma unroll
        for (int j = 0; j < kStatsMaxRowsPerLane; ++j) {
            const int b = lane + 32 * j;
            vp[j] = b < nblk ? part_p[int64_t(e) * nblk + b] : 0.f;
            vc[j] = b < nblk ? part_c[int64_t(e) * nblk + b] : 0;
        }
        double pm = 0.0, cnt = 0.0;
#pragma unroll
        for (int j = 0; j < kStatsMaxRowsPerLane; ++j) {
            pm += double(vp[j]);
            cnt += double(vc[j]);
        }
        pm = warp_sum_fixed(pm) / double(T);
        const double frac = warp_sum_fixed(cnt) / double(T);
        if (lane == 0) {
            term[e] = frac * pm;
            if (expert_stats) {
                expert_stats[e] = float(frac);
                expert_stats[E + e] = float(pm);
            }
        }
    }
    __syncthreads();
    if (w == 0) {
        double bal = 0.0, sc[3] = {0.0, 0.0, 0.0};
        for (int e = lane; e < E; e += 32) bal += term[e];
        float vs[kStatsMaxRowsPerLane][3];
#pragma unroll
        for (int jb = 0; jb < kStatsMaxRowsPerLane; ++jb) {
            const int b = lane + 32 * jb;
#pragma unroll
            for (int j = 0; j < 3; ++j) vs[jb][j] = b < nblk ? part_s[b * 3 + j] : 0.f;
        }
#pragma unroll
        for (int jb = 0; jb < kStatsMaxRowsPerLane; ++jb)
#pragma unroll
            for (int j = 0; j < 3; ++j) sc[j] += double(vs[jb][j]);
        bal = warp_sum_fixed(bal) * double(E);
        for (int j = 0; j < 3; ++j) sc[j] = warp_sum_fixed(sc[j]);
        if (lane == 0) {
            const double z = sc[2] / double(T);
            stats[0] = float(sc[0] / double(T));
            stats[1] = float(sc[1] / double(T));
            stats[2] = float(bal);
            stats[3] = float(z);
            stats[4] = float(bal + double(z_weight) * z);
        }
    }
}
}  // namespace

// Blocks of the telemetry kernel: a warp per token up to the most partial rows
// the final sum reads (32 x kStatsMaxRowsPerLane); larger batches loop.
int route_stats_blocks(int T) {
    const int need = (T + kStatsWarps - 1) / kStatsWarps;
    const int cap = 32 * kStatsMaxRowsPerLane;
    return need < cap ? need : cap;
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
        const cudaError_t le = launch_pdl(pdl, route_stats_final, dim3(1), dim3(1024), 0, stream, part_p, part_c,
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

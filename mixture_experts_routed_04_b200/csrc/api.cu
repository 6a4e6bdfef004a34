// api.cu — the C ABI declared in include/moe.h: parameter checks, workspace
// layout, and the order of launches. Every step of the layer runs in the
// kernels of this library; nothing here computes on the host beyond sizes.
#include <atomic>
#include <cmath>
#include <cstring>

#include "internal.h"

namespace moe {

cudaError_t launch_schedule(const Dims& D, const int32_t* offsets, int32_t* tile_base, int32_t* stream_list,
                            int32_t* n_stream, uint32_t* err, cudaStream_t s);
cudaError_t launch_gather(const Dims& D, const uint16_t* x, const int32_t* sorted_token, const int32_t* offsets,
                          uint16_t* xg, uint32_t* err, cudaStream_t s);
cudaError_t launch_scatter_rows(const Dims& D, const uint16_t* x, const int32_t* pair_row, const int32_t* offsets,
                                uint16_t* xg, uint32_t* err, cudaStream_t s);
cudaError_t launch_tensor_ffn(const Dims& D, const uint16_t* xg, uint16_t* h, const int32_t* tile_base,
                              const int32_t* offsets, const int32_t* sorted_pair, const float* topk_w,
                              const moe_weights* w,
                              uint16_t* y_rows, int32_t* counters, uint32_t* err, uint64_t wait_ns,
                              const uint16_t* x_fused, const int32_t* sorted_token, cudaStream_t s);
cudaError_t launch_convert_bf16_f16(const uint16_t* src, uint16_t* dst, int64_t n, uint32_t* err, cudaStream_t s);
cudaError_t launch_stream_ffn(const Dims& D, const uint16_t* xg, uint16_t* h, float* part, const int32_t* offsets,
                              const int32_t* stream_list, const int32_t* n_stream, const int32_t* sorted_pair,
                              const float* topk_w, const moe_weights* w, uint16_t* y_rows, uint32_t* err,
                              uint64_t wait_ns, const CombineArgs* comb, cudaStream_t s);

static std::atomic<uint64_t> g_wait_ns{1000000000ull};

int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!cached[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}

static size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Host-side checks of moe_params; fills D. Returns MOE_OK or an error code.
int make_dims(const moe_params* p, Dims* D) {
    if (!p || !D) return MOE_ERR_INVALID_ARG;
    // T = 0 (an empty batch) is valid: the calls launch nothing and report empty results
    if (p->T < 0 || p->E < 1 || p->E > kMaxE || p->k < 1 || p->k > kMaxK || p->k > p->E) return MOE_ERR_INVALID_ARG;
    if (p->d_model < 64 || p->d_model % 64 || p->d_ff < 64 || p->d_ff % 64) return MOE_ERR_INVALID_ARG;
    if (!(p->capacity_factor >= 0.f) || !std::isfinite(p->capacity_factor)) return MOE_ERR_INVALID_ARG;
    if (!std::isfinite(p->swiglu_limit)) return MOE_ERR_INVALID_ARG;
    if (p->weight_format != MOE_WEIGHTS_BF16 && p->weight_format != MOE_WEIGHTS_Q4G32) return MOE_ERR_INVALID_ARG;
    if (p->variant < MOE_VARIANT_AUTO || p->variant > MOE_VARIANT_STREAM) return MOE_ERR_INVALID_ARG;
    if (p->has_shared != 0 && p->has_shared != 1) return MOE_ERR_INVALID_ARG;
    if (p->out_dtype != MOE_OUT_F32 && p->out_dtype != MOE_OUT_BF16) return MOE_ERR_INVALID_ARG;
    if (p->down_dtype != MOE_DOWN_BF16 && p->down_dtype != MOE_DOWN_F16) return MOE_ERR_INVALID_ARG;
    if (p->down_dtype == MOE_DOWN_F16 && p->weight_format != MOE_WEIGHTS_BF16) return MOE_ERR_INVALID_ARG;
    if (p->tile_ctas < MOE_TILE_AUTO || p->tile_ctas > MOE_TILE_PAIR) return MOE_ERR_INVALID_ARG;
    const int64_t pairs = int64_t(p->T) * p->k;
    if (pairs + p->T >= (int64_t(1) << 31)) return MOE_ERR_INVALID_ARG;
    if (int64_t(p->d_model) * p->d_ff * p->E >= (int64_t(1) << 40)) return MOE_ERR_INVALID_ARG;
    if (p->has_shared && (p->d_ff_shared != p->d_ff)) return MOE_ERR_UNSUPPORTED;
    if (p->weight_format == MOE_WEIGHTS_Q4G32 && (p->has_shared || p->variant == MOE_VARIANT_STREAM))
        return MOE_ERR_UNSUPPORTED;  // Q4G32 runs on the tcgen05 tile kernels only
    D->T = p->T;
    D->d = p->d_model;
    D->f = p->d_ff;
    D->E = p->E;
    D->k = p->k;
    D->has_shared = p->has_shared;
    D->Etot = p->E + p->has_shared;
    D->pairs = pairs;
    D->cap = -1;
    int64_t routed_rows = pairs;
    if (p->capacity_factor > 0.f) {
        const double c = std::ceil(double(p->capacity_factor) * double(p->T) * double(p->k) / double(p->E));
        if (c < 0 || c > double(1 << 30)) return MOE_ERR_INVALID_ARG;
        D->cap = int(c);
        const int64_t lim = int64_t(D->cap) * p->E;
        if (lim < routed_rows) routed_rows = lim;
    }
    D->rows = routed_rows + (p->has_shared ? p->T : 0);
    if (D->rows < 1) D->rows = 1;
    const int64_t ppb = int64_t(kPermWarps) * 32 * perm_rounds(pairs);  // pairs per permutation block
    D->perm_blocks = int((pairs + ppb - 1) / ppb);
    D->fmt = p->weight_format;
    D->variant = p->variant;
    // Default variant choice from the measured table (kStreamTable): the
    // touched experts' gate/up tiles (at most min(E', pairs') experts) against
    // the SM count picks the largest expert that still streams.
    if (p->stream_max_rows < 0) {
        const int64_t touched_max = std::min<int64_t>(p->E + p->has_shared, pairs + p->has_shared);
        const double ratio = double(touched_max * ((p->d_ff + 127) / 128)) / double(num_sms());
        D->stream_max_rows = 0;
        for (int i = 0; i < kStreamTableRows; ++i)
            if (ratio < double(kStreamTable[i].tiles_per_sm)) {
                D->stream_max_rows = kStreamTable[i].max_rows;
                break;
            }
    } else {
        D->stream_max_rows = p->stream_max_rows;
    }
    D->limit = p->swiglu_limit;
    D->out_bf16 = p->out_dtype == MOE_OUT_BF16;
    D->down_f16 = p->down_dtype == MOE_DOWN_F16;
    // SM pairs on 256-row tiles (bf16 weights only) on request. Not the
    // default: on the 4096-token prompt layer (experts of 26 to 3017 rows,
    // median 101) the pairs round the rows up 1.63x against 1.09x for one SM
    // per 128-row tile, and measured slower on B200.
    D->tile_pair = p->weight_format == MOE_WEIGHTS_BF16 && p->tile_ctas == MOE_TILE_PAIR;
    // The streaming kernels take bf16 weights only (Q4G32 runs on the tiles).
    if (p->weight_format != MOE_WEIGHTS_BF16) D->stream_max_rows = 0;
    // K split of the streaming gate/up, for load balance only: when few experts
    // are touched (decode), split d so that there are a few work items per SM
    // (the slices stay multiples of 64).
    int ks = 1;
    const int64_t touched = std::min<int64_t>(D->Etot, pairs + p->has_shared);
    const int64_t units = touched * (p->d_ff / 64);
    const int64_t sms = num_sms();
    while (ks < 8 && units * ks < 4 * sms && (p->d_model % (ks * 2 * 64)) == 0) ks *= 2;
    D->ks = ks;
    return MOE_OK;
}

WsLayout ws_layout(const Dims& D, int which) {
    WsLayout L;
    std::memset(&L, 0, sizeof(L));
    size_t off = 256;  // [0, 256): error word
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    const bool fwd = which == MOE_WS_FORWARD || which == MOE_WS_FORWARD_HOST;
    const bool perm = which == MOE_WS_PERMUTE || fwd;
    const bool ffn = which == MOE_WS_EXPERT_FFN || fwd;
    if (which == MOE_WS_BACKWARD) {
        const int64_t rp = bwd_padded_rows(D);
        const int nt = (D.f + 255) / 256;
        L.b_poff = take(size_t(D.Etot + 1) * 4);
        L.b_tile_base = take(size_t(D.Etot + 1) * 4);
        L.b_wbase = take(size_t(D.Etot + 1) * 4);
        L.b_counters = take(8 * 4);
        L.b_xg = take(size_t(rp) * D.d * 2);
        L.b_xg16 = take(size_t(rp) * D.d * 2);
        L.b_dog = take(size_t(rp) * D.d * 2);
        L.b_gu = take(size_t(rp) * 2 * D.f * 2);
        L.b_hw = take(size_t(rp) * D.f * 2);
        L.b_dgu = take(size_t(rp) * 2 * D.f * 2);
        L.b_dgu16 = take(size_t(rp) * 2 * D.f * 2);
        L.b_dxr = take(size_t(D.rows) * D.d * 2);
        L.b_dwp = take(size_t(D.rows) * nt * 2 * 4);
    }
    if (which == MOE_WS_ROUTE_STATS) {
        const int nb = route_stats_blocks(D.T > 0 ? D.T : 1);
        L.stats_p = take(size_t(nb) * D.E * 4);
        L.stats_c = take(size_t(nb) * D.E * 4);
        L.stats_s = take(size_t(nb) * 3 * 4);
    }
    if (perm) {
        L.blockcounts = take(size_t(D.perm_blocks) * D.E * 4);
        L.blockbase = take(size_t(D.perm_blocks) * D.E * 4);
    }
    if (ffn) {
        L.tile_base = take(size_t(D.Etot + 1) * 2 * 4);  // 128-row and 256-row tile prefixes
        L.stream_list = take(size_t(D.Etot) * 4);
        L.n_stream = take(16);  // [0] streaming experts, [1], [2] tile-unit counters
        L.xg = take(size_t(D.rows) * D.d * 2);
        L.h = take(size_t(D.rows) * D.f * 2);
        if (D.ks > 1) L.part = take(size_t(D.ks) * 2 * D.rows * D.f * 4);
    }
    if (fwd) {
        L.topk_idx = take(size_t(D.pairs) * 4);
        L.topk_w = take(size_t(D.pairs) * 4);
        L.counts = take(size_t(D.Etot) * 4);
        L.kept = take(size_t(D.Etot) * 4);
        L.offsets = take(size_t(D.Etot + 1) * 4);
        L.sorted_token = take(size_t(D.rows) * 4);
        L.sorted_pair = take(size_t(D.rows) * 4);
        L.pair_row = take(size_t(D.pairs) * 4);
        L.y_rows = take(size_t(D.rows) * D.d * 2);
        L.comb = take(size_t(combine_blocks(D)) * 4);
    }
    if (which == MOE_WS_FORWARD_HOST) {
        L.x_dev = take(size_t(D.T) * D.d * 2);
        L.logits_dev = take(size_t(D.T) * D.E * 4);
        L.out_dev = take(size_t(D.T) * D.d * (D.out_bf16 ? 2 : 4));
    }
    L.total = off;
    return L;
}

// Whether any expert can take the tcgen05 tiles. An expert holds at most T rows
// (a token's k experts are distinct; the shared expert holds exactly T), so
// with T <= stream_max_rows the automatic choice streams every expert and the
// two persistent GEMMs would only start and exit: they are not launched.
// Whether the weight-streaming kernels run: every expert with a forced
// MOE_VARIANT_STREAM, else the experts of at most stream_max_rows rows.
static bool streams(const Dims& D) {
    return D.variant == MOE_VARIANT_STREAM || (D.variant == MOE_VARIANT_AUTO && D.stream_max_rows > 0);
}

static bool tiles_needed(const Dims& D) {
    if (D.variant == MOE_VARIANT_STREAM) return false;
    if (D.variant == MOE_VARIANT_AUTO && D.stream_max_rows > 0 && D.T <= D.stream_max_rows) return false;
    return true;
}

// moe_forward of at most kCombFuseMaxTokens tokens whose experts all stream: the
// streaming down kernel does the combine (its last arrival on each 256-column
// block sums that block), so the combine launch is not made.
static bool combine_fused(const Dims& D) {
    return D.T <= kFrontMaxTokens && D.T <= kCombFuseMaxTokens && streams(D) && !tiles_needed(D);
}

// x small enough to stay in L2 while the rows are gathered.
static bool x_in_l2(const Dims& D) { return int64_t(D.T) * D.d * 2 <= (int64_t(64) << 20); }

// The bf16 gate/up on one SM per tile gathers its rows itself (no gather kernel)
// when x sits in L2 and no expert streams (the streaming kernels read the
// gathered copy).
static bool gather_fused(const Dims& D) {
    const bool streaming = streams(D);
    return kFusedGather && D.fmt == MOE_WEIGHTS_BF16 && !D.tile_pair && x_in_l2(D) && !streaming && tiles_needed(D);
}

cudaError_t launch_expert_ffn(const Dims& D, const WsLayout& L, const FfnArgs& a, cudaStream_t s) {
    uint8_t* ws = a.ws;
    int32_t* tile_base = reinterpret_cast<int32_t*>(ws + L.tile_base);
    int32_t* stream_list = reinterpret_cast<int32_t*>(ws + L.stream_list);
    int32_t* n_stream = reinterpret_cast<int32_t*>(ws + L.n_stream);
    uint16_t* xg = reinterpret_cast<uint16_t*>(ws + L.xg);
    uint16_t* h = reinterpret_cast<uint16_t*>(ws + L.h);
    float* part = L.part ? reinterpret_cast<float*>(ws + L.part) : nullptr;
    cudaError_t e = cudaSuccess;
    if (!a.scheduled &&
        (e = launch_schedule(D, a.offsets, tile_base, stream_list, n_stream, a.err, s)) != cudaSuccess)
        return e;
    // Rows in expert order for both variants (fp16 for Q4G32, whose MMAs run
    // in fp16). A TMA tile::gather4 of the rows inside the GEMM was measured
    // slower: 32 TMA instructions per k-block left the producer behind.
    // moe_forward has pair_row and, when x is larger than half of L2, copies in
    // token order so that each x row is read from HBM once instead of k times
    // (Q4G32 workload: 234 against 326 us); with x in L2 the row-order gather,
    // which spreads small batches over more threads, is faster.
    const bool token_order = a.pair_row && !x_in_l2(D);
    const bool fused = gather_fused(D);
    if (!fused && !a.gathered &&
        (e = token_order ? launch_scatter_rows(D, a.x, a.pair_row, a.offsets, xg, a.err, s)
                         : launch_gather(D, a.x, a.sorted_token, a.offsets, xg, a.err, s)) != cudaSuccess)
        return e;
    if (tiles_needed(D)) {
        if ((e = launch_tensor_ffn(D, xg, h, tile_base, a.offsets, a.sorted_pair, a.topk_w, a.w, a.y_rows,
                                   n_stream + 1, a.err, a.wait_ns, fused ? a.x : nullptr, a.sorted_token, s)) !=
            cudaSuccess)
            return e;
    }
    if (streams(D)) {
        if ((e = launch_stream_ffn(D, xg, h, part, a.offsets, stream_list, n_stream, a.sorted_pair, a.topk_w, a.w,
                                   a.y_rows, a.err, a.wait_ns, a.comb, s)) != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

}  // namespace moe

using namespace moe;

static bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int check_ws(const Dims& D, int which, const void* ws, size_t ws_bytes) {
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return MOE_ERR_MISALIGNED;
    if (ws_bytes < ws_layout(D, which).total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    return MOE_OK;
}

static int check_weights(const Dims& D, const moe_weights* w) {
    if (!w || !w->w_gate || !w->w_up || !w->w_down) return MOE_ERR_INVALID_ARG;
    if (!al16(w->w_gate) || !al16(w->w_up) || !al16(w->w_down)) return MOE_ERR_MISALIGNED;
    if (D.fmt == MOE_WEIGHTS_Q4G32) {
        if (!w->s_gate || !w->s_up || !w->s_down) return MOE_ERR_INVALID_ARG;
        if (!al16(w->s_gate) || !al16(w->s_up) || !al16(w->s_down)) return MOE_ERR_MISALIGNED;
    }
    if (D.has_shared) {
        if (!w->shared_gate || !w->shared_up || !w->shared_down) return MOE_ERR_INVALID_ARG;
        if (!al16(w->shared_gate) || !al16(w->shared_up) || !al16(w->shared_down)) return MOE_ERR_MISALIGNED;
    }
    return MOE_OK;
}

static int status_of(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

extern "C" {

int moe_version(void) { return 100; }

const char* moe_status_string(int s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_MISALIGNED: return "misaligned pointer";
        case MOE_ERR_DEVICE: return "device error word set";
        default: return "unknown status";
    }
}

int moe_capacity(const moe_params* p, int32_t* cap) {
    Dims D;
    const int st = make_dims(p, &D);
    if (st != MOE_OK) return st;
    if (!cap) return MOE_ERR_INVALID_ARG;
    *cap = D.cap;
    return MOE_OK;
}

int moe_max_rows(const moe_params* p, int64_t* rows) {
    Dims D;
    const int st = make_dims(p, &D);
    if (st != MOE_OK) return st;
    if (!rows) return MOE_ERR_INVALID_ARG;
    *rows = D.rows;
    return MOE_OK;
}

int moe_tile_ctas(const moe_params* p, int32_t* ctas) {
    Dims D;
    const int st = make_dims(p, &D);
    if (st != MOE_OK) return st;
    if (!ctas) return MOE_ERR_INVALID_ARG;
    *ctas = D.tile_pair ? MOE_TILE_PAIR : MOE_TILE_ONE;
    return MOE_OK;
}

size_t moe_workspace_size(const moe_params* p, int which) {
    Dims D;
    if (make_dims(p, &D) != MOE_OK || which < MOE_WS_ROUTE || which > MOE_WS_BACKWARD) return 0;
    return ws_layout(D, which).total;
}

int moe_route(const moe_params* p, const float* logits, int32_t* topk_idx, float* topk_w, void* ws,
              size_t ws_bytes, moe_stream_t stream) {
    Dims D;
    int st = make_dims(p, &D);
    if (st != MOE_OK) return st;
    if ((st = check_ws(D, MOE_WS_ROUTE, ws, ws_bytes)) != MOE_OK) return st;
    if (D.T == 0) return MOE_OK;  // empty batch: the (empty) buffers may be null
    if (!logits || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    return status_of(launch_route(logits, D.T, D.E, D.k, topk_idx, topk_w, stream));
}

int moe_route_stats(const moe_params* p, const float* logits, int32_t* topk_idx, float* topk_w, float z_weight,
                    float* stats, float* kept_tok, int32_t* want_tok, float* expert_stats, void* ws,
                    size_t ws_bytes, moe_stream_t stream) {
    Dims D;
    int st = make_dims(p, &D);
    if (st != MOE_OK) return st;
    if ((st = check_ws(D, MOE_WS_ROUTE_STATS, ws, ws_bytes)) != MOE_OK) return st;
    if (D.T == 0) return MOE_OK;
    if (!logits || !topk_idx || !topk_w || !stats || !std::isfinite(z_weight)) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(D, MOE_WS_ROUTE_STATS);
    uint8_t* w = static_cast<uint8_t*>(ws);
    return status_of(launch_route_stats(logits, D.T, D.E, D.k, topk_idx, topk_w, z_weight, stats, kept_tok,
                                        want_tok, expert_stats, reinterpret_cast<float*>(w + L.stats_p),
                                        reinterpret_cast<int32_t*>(w + L.stats_c),
                                        reinterpret_cast<float*>(w + L.stats_s), stream));
}

int moe_permute(const moe_params* p, const int32_t* topk_idx, int32_t* counts, int32_t* kept_counts,
                int32_t* offsets, int32_t* sorted_token, int32_t* sorted_pair, int32_t* pair_row, void* ws,
                size_t ws_bytes, moe_stream_t stream) {
    Dims D;
    int st = make_dims(p, &D);
    if (st != MOE_OK) return st;
    if ((st = check_ws(D, MOE_WS_PERMUTE, ws, ws_bytes)) != MOE_OK) return st;
    if (!topk_idx || !counts || !kept_counts || !offsets || !sorted_token || !sorted_pair || !pair_row)
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(D, MOE_WS_PERMUTE);
    uint8_t* w = static_cast<uint8_t*>(ws);
    return status_of(launch_permute(D, topk_idx, reinterpret_cast<int32_t*>(w + L.blockcounts),
                                    reinterpret_cast<int32_t*>(w + L.blockbase), counts, kept_counts, offsets,
                                    sorted_token, sorted_pair, pair_row, reinterpret_cast<uint32_t*>(w), stream));
}

int moe_expert_ffn(const moe_params* p, const uint16_t* x, const int32_t* offsets, const int32_t* sorted_token,
                   const int32_t* sorted_pair, const float* topk_w, const moe_weights* w, uint16_t* y_rows,
                   void* ws, size_t ws_bytes, moe_stream_t stream) {
    Dims D;
    int st = make_dims(p, &D);
    if (st != MOE_OK) return st;
    if ((st = check_ws(D, MOE_WS_EXPERT_FFN, ws, ws_bytes)) != MOE_OK) return st;
    if (D.T == 0) return MOE_OK;
    if ((st = check_weights(D, w)) != MOE_OK) return st;
    if (!x || !offsets || !sorted_token || !sorted_pair || !topk_w || !y_rows) return MOE_ERR_INVALID_ARG;
    if (!al16(x) || !al16(y_rows)) return MOE_ERR_MISALIGNED;
    const WsLayout L = ws_layout(D, MOE_WS_EXPERT_FFN);
    FfnArgs a{x, offsets, sorted_token, sorted_pair, topk_w, w, y_rows, static_cast<uint8_t*>(ws),
              static_cast<uint32_t*>(ws), g_wait_ns.load(), false, nullptr};
    return status_of(launch_expert_ffn(D, L, a, stream));
}

int moe_combine(const moe_params* p, const uint16_t* y_rows, const int32_t* pair_row, const int32_t* offsets,
                void* out, void* ws, size_t ws_bytes, moe_stream_t stream) {
    Dims D;
    int st = make_dims(p, &D);
    if (st != MOE_OK) return st;
    if ((st = check_ws(D, MOE_WS_COMBINE, ws, ws_bytes)) != MOE_OK) return st;
    if (D.T == 0) return MOE_OK;
    if (!y_rows || !pair_row || !out || (D.has_shared && !offsets)) return MOE_ERR_INVALID_ARG;
    if (!al16(y_rows) || !al16(out)) return MOE_ERR_MISALIGNED;
    return status_of(launch_combine(D, y_rows, pair_row, offsets, out, stream));
}

static int forward_impl(const Dims& D, const WsLayout& L, const uint16_t* x, const float* logits,
                        const moe_weights* w, void* out, int32_t* counts_out, uint8_t* ws,
                        cudaStream_t stream) {
    int32_t* topk_idx = reinterpret_cast<int32_t*>(ws + L.topk_idx);
    float* topk_w = reinterpret_cast<float*>(ws + L.topk_w);
    int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
    int32_t* kept = reinterpret_cast<int32_t*>(ws + L.kept);
    int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
    int32_t* sorted_token = reinterpret_cast<int32_t*>(ws + L.sorted_token);
    int32_t* sorted_pair = reinterpret_cast<int32_t*>(ws + L.sorted_pair);
    int32_t* pair_row = reinterpret_cast<int32_t*>(ws + L.pair_row);
    uint16_t* y_rows = reinterpret_cast<uint16_t*>(ws + L.y_rows);
    uint32_t* err = reinterpret_cast<uint32_t*>(ws);
    const bool front = D.T <= kFrontMaxTokens;
    const bool fuse_comb = combine_fused(D);
    const CombineArgs comb{reinterpret_cast<int32_t*>(ws + L.comb), pair_row, out};
    cudaError_t e;
    if (front) {  // routing, permutation and schedule in one small kernel
        e = launch_front_small(D, logits, topk_idx, topk_w, counts, kept, offsets, sorted_token, sorted_pair,
                               pair_row, reinterpret_cast<int32_t*>(ws + L.tile_base),
                               reinterpret_cast<int32_t*>(ws + L.stream_list),
                               reinterpret_cast<int32_t*>(ws + L.n_stream), x,
                               front_gathers(D) ? reinterpret_cast<uint16_t*>(ws + L.xg) : nullptr,
                               fuse_comb ? comb.count : nullptr, err, stream);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    } else {
        e = launch_route(logits, D.T, D.E, D.k, topk_idx, topk_w, stream);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        // the permutation's scan also writes the tile schedule
        const ScheduleArgs sa{reinterpret_cast<int32_t*>(ws + L.tile_base),
                              reinterpret_cast<int32_t*>(ws + L.stream_list),
                              reinterpret_cast<int32_t*>(ws + L.n_stream), D.variant, D.stream_max_rows};
        e = launch_permute(D, topk_idx, reinterpret_cast<int32_t*>(ws + L.blockcounts),
                           reinterpret_cast<int32_t*>(ws + L.blockbase), counts, kept, offsets, sorted_token,
                           sorted_pair, pair_row, err, stream, &sa);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    FfnArgs a{x, offsets, sorted_token, sorted_pair, topk_w, w, y_rows, ws, err, g_wait_ns.load(), true, pair_row,
              front && front_gathers(D), fuse_comb ? &comb : nullptr};
    if ((e = launch_expert_ffn(D, L, a, stream)) != cudaSuccess) return MOE_ERR_CUDA;
    if (!fuse_comb && (e = launch_combine(D, y_rows, pair_row, offsets, out, stream)) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (counts_out &&
        cudaMemcpyAsync(counts_out, counts, size_t(D.Etot) * 4, cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

int moe_forward(const moe_params* p, const uint16_t* x, const float* logits, const moe_weights* w, void* out,
                int32_t* counts_out, void* ws, size_t ws_bytes, moe_stream_t stream) {
    Dims D;
    int st = make_dims(p, &D);
    if (st != MOE_OK) return st;
    if ((st = check_ws(D, MOE_WS_FORWARD, ws, ws_bytes)) != MOE_OK) return st;
    if (D.T == 0) {  // empty batch: nothing to read or write but the (optional) counts
        if (counts_out && cudaMemsetAsync(counts_out, 0, size_t(D.Etot) * 4, stream) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if ((st = check_weights(D, w)) != MOE_OK) return st;
    if (!x || !logits || !out) return MOE_ERR_INVALID_ARG;
    if (!al16(x) || !al16(out)) return MOE_ERR_MISALIGNED;
    return forward_impl(D, ws_layout(D, MOE_WS_FORWARD), x, logits, w, out, counts_out, static_cast<uint8_t*>(ws),
                        stream);
}

static int forward_host_impl(const moe_params* p, const uint16_t* x_host, const float* logits_host,
                             const moe_weights* w, void* out_host, void* ws, size_t ws_bytes, moe_stream_t stream,
                             bool sync) {
    Dims D;
    int st = make_dims(p, &D);
    if (st != MOE_OK) return st;
    if ((st = check_ws(D, MOE_WS_FORWARD_HOST, ws, ws_bytes)) != MOE_OK) return st;
    if (D.T == 0) return MOE_OK;
    if ((st = check_weights(D, w)) != MOE_OK) return st;
    if (!x_host || !logits_host || !out_host) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(D, MOE_WS_FORWARD_HOST);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    uint16_t* xd = reinterpret_cast<uint16_t*>(wsb + L.x_dev);
    float* ld = reinterpret_cast<float*>(wsb + L.logits_dev);
    void* od = wsb + L.out_dev;
    if (cudaMemcpyAsync(xd, x_host, size_t(D.T) * D.d * 2, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(ld, logits_host, size_t(D.T) * D.E * 4, cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    st = forward_impl(D, L, xd, ld, w, od, nullptr, wsb, stream);
    if (st != MOE_OK) return st;
    if (cudaMemcpyAsync(out_host, od, size_t(D.T) * D.d * (D.out_bf16 ? 2 : 4), cudaMemcpyDeviceToHost, stream) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    if (!sync) return MOE_OK;
    return cudaStreamSynchronize(stream) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_forward_host(const moe_params* p, const uint16_t* x_host, const float* logits_host, const moe_weights* w,
                     void* out_host, void* ws, size_t ws_bytes, moe_stream_t stream) {
    return forward_host_impl(p, x_host, logits_host, w, out_host, ws, ws_bytes, stream, true);
}

int moe_forward_host_async(const moe_params* p, const uint16_t* x_host, const float* logits_host,
                           const moe_weights* w, void* out_host, void* ws, size_t ws_bytes, moe_stream_t stream) {
    return forward_host_impl(p, x_host, logits_host, w, out_host, ws, ws_bytes, stream, false);
}

int moe_expert_ffn_backward(const moe_params* p, const uint16_t* x, const int32_t* topk_idx, const float* topk_w,
                            const int32_t* offsets, const int32_t* sorted_token, const int32_t* sorted_pair,
                            const int32_t* pair_row, const moe_weights* w, const float* dout, const moe_grads* g,
                            void* ws, size_t ws_bytes, moe_stream_t stream) {
    Dims D;
    int st = make_dims(p, &D);
    if (st != MOE_OK) return st;
    // bf16 gate/up weights and the fp16 copy of W_down (moe_convert_bf16_to_f16)
    if (D.fmt != MOE_WEIGHTS_BF16 || !D.down_f16) return MOE_ERR_UNSUPPORTED;
    if ((st = check_ws(D, MOE_WS_BACKWARD, ws, ws_bytes)) != MOE_OK) return st;
    if (D.T == 0) return MOE_OK;
    if ((st = check_weights(D, w)) != MOE_OK) return st;
    if (!x || !topk_w || !offsets || !sorted_token || !sorted_pair || !pair_row || !dout || !g) return MOE_ERR_INVALID_ARG;
    if (!g->dx || !g->dw_gate || !g->dw_up || !g->dw_down || !g->d_topk_w) return MOE_ERR_INVALID_ARG;
    if (g->dlogits && !topk_idx) return MOE_ERR_INVALID_ARG;
    if (D.has_shared && (!g->dshared_gate || !g->dshared_up || !g->dshared_down)) return MOE_ERR_INVALID_ARG;
    if (!al16(x) || !al16(dout) || !al16(g->dx) || !al16(g->dw_gate) || !al16(g->dw_up) || !al16(g->dw_down))
        return MOE_ERR_MISALIGNED;
    if (D.has_shared && (!al16(g->dshared_gate) || !al16(g->dshared_up) || !al16(g->dshared_down)))
        return MOE_ERR_MISALIGNED;
    BwdArgs a{x, dout, topk_idx, topk_w, offsets, sorted_token, sorted_pair, pair_row, w, g,
              static_cast<uint8_t*>(ws), ws_layout(D, MOE_WS_BACKWARD), static_cast<uint32_t*>(ws),
              g_wait_ns.load()};
    return status_of(launch_backward(D, a, stream));
}

int moe_variant_table(float* tiles_per_sm, int32_t* max_rows, int n) {
    if (n < 0 || (n > 0 && (!tiles_per_sm || !max_rows))) return -1;
    for (int i = 0; i < kStreamTableRows && i < n; ++i) {
        tiles_per_sm[i] = kStreamTable[i].tiles_per_sm;
        max_rows[i] = kStreamTable[i].max_rows;
    }
    return kStreamTableRows;
}

int moe_get_error(const void* ws, uint32_t* err, moe_stream_t stream) {
    if (!ws || !err) return MOE_ERR_INVALID_ARG;
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, stream) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
    *err = v;
    return v ? MOE_ERR_DEVICE : MOE_OK;
}

int moe_clear_error(void* ws, moe_stream_t stream) {
    if (!ws) return MOE_ERR_INVALID_ARG;
    return cudaMemsetAsync(ws, 0, 4, stream) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_launch_count(const moe_params* p, int which, int* n) {
    Dims D;
    const int st = make_dims(p, &D);
    if (st != MOE_OK) return st;
    if (!n || which < MOE_WS_ROUTE || which > MOE_WS_BACKWARD) return MOE_ERR_INVALID_ARG;
    if (D.T == 0) {
        *n = 0;
        return MOE_OK;
    }
    int ffn = 1;  // schedule
    if (!gather_fused(D)) ffn += 1;                 // gather
    if (tiles_needed(D)) ffn += 2;                  // two tcgen05 GEMMs
    if (streams(D)) ffn += 2 + (D.ks > 1 && !stream_fold(D) ? 1 : 0);  // + the K-split reduce
    switch (which) {
        case MOE_WS_ROUTE: *n = 1; break;
        case MOE_WS_PERMUTE: *n = 3; break;
        case MOE_WS_EXPERT_FFN: *n = ffn; break;
        case MOE_WS_COMBINE: *n = 1; break;
        case MOE_WS_ROUTE_STATS: *n = 2; break;
        // schedule, gather, 6 GEMMs, zeroing, combine, routing-weight reduce, and the routing
        // backward (when dlogits is asked for; 11 without)
        case MOE_WS_BACKWARD: *n = 12; break;
        // moe_forward: the front kernel(s) write the schedule, so the expert FFN's own
        // schedule launch is not made (nor, for the smallest batches, the gather, and
        // when the streaming down kernel combines, the combine); nor, when the scatter
        // blocks form the scan themselves, the permutation's scan launch
        default:
            *n = D.T <= kFrontMaxTokens
                     ? 1 + (ffn - 1) - (front_gathers(D) && !gather_fused(D) ? 1 : 0) + (combine_fused(D) ? 0 : 1)
                     : 1 + (perm_scan_fused(D) ? 2 : 3) + (ffn - 1) + 1;
            break;
    }
    return MOE_OK;
}

int moe_convert_bf16_to_f16(const uint16_t* src, uint16_t* dst, int64_t n, void* err_ws, moe_stream_t stream) {
    if (n < 0 || (n > 0 && (!src || !dst))) return MOE_ERR_INVALID_ARG;
    if (!al16(src) || !al16(dst)) return MOE_ERR_MISALIGNED;
    if (err_ws && (reinterpret_cast<uintptr_t>(err_ws) & 255u)) return MOE_ERR_MISALIGNED;
    return status_of(launch_convert_bf16_f16(src, dst, n, static_cast<uint32_t*>(err_ws), stream));
}

int moe_set_wait_limit_ns(uint64_t ns) {
    g_wait_ns.store(ns ? ns : 1000000000ull);
    return MOE_OK;
}

}  // extern "C"

// internal.h — launchers and workspace layout shared by the kernel files and the C ABI.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kMaxE = 256;
constexpr int kMaxK = 8;
constexpr int kPermWarps = 8;                         // warps per permutation block
// Rounds of 32 pairs per permutation warp: 2 (512-pair blocks) spread prompt-sized
// batches over more SMs; above kPermSmallPairs pairs, 8 (2048-pair blocks) keep the
// scan over the blocks short.
constexpr int kPermRoundsSmall = 2, kPermRoundsLarge = 8;
constexpr int64_t kPermSmallPairs = 65536;
inline int perm_rounds(int64_t pairs) { return pairs <= kPermSmallPairs ? kPermRoundsSmall : kPermRoundsLarge; }
constexpr int kPermMaxPairsPerBlock = kPermWarps * 32 * kPermRoundsLarge;
// moe_forward's permutation without its scan launch: each scatter block copies the
// per-block counts ([blocks][E], at most this many bytes) into shared memory and forms
// its own bases and the expert offsets; block 0 writes counts, kept, offsets and the
// tile schedule (one thread per expert: Etot <= the block's 256 threads).
constexpr int kScanFusedMaxBytes = 96 * 1024;
constexpr int kTileM = 128;                           // rows per tcgen05 tile
// AUTO variant choice, measured on B200 (decode-shaped layers, d=4096, f=1536,
// E=256 + shared, whose routing gives `touched` experts the same rows each;
// every expert on the tcgen05 tiles against every routed expert streaming):
// experts of at most max_rows kept rows take the weight-streaming kernels while
// the touched experts' gate/up tiles number fewer than tiles_per_sm x SMs; the
// first matching row applies; past the last row every expert takes the tiles.
struct StreamRule {
    float tiles_per_sm;
    int max_rows;
};
constexpr StreamRule kStreamTable[] = {{1.5f, 4}, {2.5f, 1}};
constexpr int kStreamTableRows = int(sizeof(kStreamTable) / sizeof(kStreamTable[0]));

// Everything a call derives from moe_params on the host.
struct Dims {
    int T, d, f, E, k, Etot;  // Etot = E + has_shared
    int has_shared;
    int cap;                  // -1: no cap
    int64_t rows;             // rows of the permuted buffers
    int64_t pairs;            // T * k
    int perm_blocks;          // blocks of the permutation kernels
    int fmt, variant, stream_max_rows;
    float limit;
    int ks;                   // K-split of the streaming gate/up kernel
    int out_bf16;             // layer output in bf16 (else fp32)
    int down_f16;             // W_down given as fp16 (prepared at load time)
    int tile_pair;            // bf16 tcgen05 GEMMs on SM pairs (256-row tiles)
};
inline bool perm_scan_fused(const Dims& D) {
    return D.Etot <= kPermWarps * 32 && int64_t(D.perm_blocks) * D.E * 4 <= kScanFusedMaxBytes;
}

// Byte offsets of every scratch array inside a workspace (0 = absent).
struct WsLayout {
    size_t err;                                    // uint32 error word (always at 0)
    size_t blockcounts, blockbase;                 // permute: int32 [perm_blocks, E]
    size_t tile_base, stream_list, n_stream;       // expert_ffn schedule
    size_t xg, h, part;                            // expert_ffn: gathered x, h, split-K partials
    size_t topk_idx, topk_w, counts, kept, offsets, sorted_token, sorted_pair, pair_row, y_rows;  // forward
    size_t comb;                                   // forward: fused-combine arrival counters
    size_t x_dev, logits_dev, out_dev;             // forward_host
    size_t stats_p, stats_c, stats_s;              // route_stats: per-block partial sums
    // backward (padded row space, see backward.cu)
    size_t b_poff, b_tile_base, b_wbase, b_counters, b_xg, b_xg16, b_dog, b_gu, b_hw, b_dgu, b_dgu16, b_dxr, b_dwp;
    size_t total;
};

WsLayout ws_layout(const Dims& D, int which);

// The parameter checks every entry point shares: fills D from moe_params and
// returns MOE_OK, or the status the entry point returns unchanged.
int make_dims(const moe_params* p, Dims* D);

// ---- launchers (all asynchronous on `s`)
cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* topk_idx, float* topk_w,
                         cudaStream_t s);

int route_stats_blocks(int T);
// The streaming down kernel sums the K-split gate/up partials itself (stream.cu).
bool stream_fold(const Dims& D);
cudaError_t launch_route_stats(const float* logits, int T, int E, int k, int32_t* topk_idx, float* topk_w,
                               float z_weight, float* stats, float* kept_tok, int32_t* want_tok,
                               float* expert_stats, float* part_p, int32_t* part_c, float* part_s,
                               cudaStream_t stream);

// The tile schedule (K3), when the permutation's scan kernel runs it too
// (moe_forward with more than kFrontMaxTokens tokens).
struct ScheduleArgs {
    int32_t* tile_base;
    int32_t* stream_list;
    int32_t* n_stream;
    int variant, stream_max;
};
cudaError_t launch_permute(const Dims& D, const int32_t* topk_idx, int32_t* blockcounts, int32_t* blockbase,
                           int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* sorted_token,
                           int32_t* sorted_pair, int32_t* pair_row, uint32_t* err, cudaStream_t s,
                           const ScheduleArgs* sched = nullptr);

// Batches of at most this many tokens run routing, permutation and the tile
// schedule as one fused single-block kernel (front.cu).
constexpr int kFrontMaxTokens = 64;
// The fused front kernel also gathers the rows (bf16) when at most this many bytes of
// rows can result: one block copies them faster than a separate launch starts.
constexpr int64_t kFrontGatherBytes = 96 << 10;
bool front_gathers(const Dims& D);
// x / xg: the rows to gather and their destination when front_gathers(D), else null.
// comb_count: the fused combine's counters to zero (combine_blocks(D) of them), or null.
cudaError_t launch_front_small(const Dims& D, const float* logits, int32_t* topk_idx, float* topk_w,
                               int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* sorted_token,
                               int32_t* sorted_pair, int32_t* pair_row, int32_t* tile_base, int32_t* stream_list,
                               int32_t* n_stream, const uint16_t* x, uint16_t* xg, int32_t* comb_count,
                               uint32_t* err, cudaStream_t s);

// The bf16 gate/up GEMM gathers its rows from x itself (no gathered copy).
constexpr bool kFusedGather = false;

// moe_forward of a few tokens whose experts all stream: the streaming down kernel
// also does the combine (stream.cu); count: [combine_blocks(D)] int32, zeroed by the
// front kernel.
struct CombineArgs {
    int32_t* count;
    const int32_t* pair_row;
    void* out;
};
constexpr int kCombFuseMaxTokens = 2;
inline int combine_blocks(const Dims& D) { return (D.d + 255) / 256; }

struct FfnArgs {
    const uint16_t* x;
    const int32_t* offsets;
    const int32_t* sorted_token;
    const int32_t* sorted_pair;
    const float* topk_w;
    const moe_weights* w;
    uint16_t* y_rows;
    uint8_t* ws;
    uint32_t* err;
    uint64_t wait_ns;
    bool scheduled;            // the front kernels already wrote the tile schedule
    const int32_t* pair_row;   // moe_forward: row of each pair (-1 dropped), for the token-order row copy
    bool gathered = false;     // the front kernel already wrote the gathered rows
    const CombineArgs* comb = nullptr;  // the streaming down kernel also combines
};
cudaError_t launch_expert_ffn(const Dims& D, const WsLayout& L, const FfnArgs& a, cudaStream_t s);

cudaError_t launch_combine(const Dims& D, const uint16_t* y_rows, const int32_t* pair_row, const int32_t* offsets,
                           void* out, cudaStream_t s);

// Backward of the expert FFN (backward.cu).
struct BwdArgs {
    const uint16_t* x;
    const float* dout;
    const int32_t* topk_idx;
    const float* topk_w;
    const int32_t* offsets;
    const int32_t* sorted_token;
    const int32_t* sorted_pair;
    const int32_t* pair_row;
    const moe_weights* w;
    const moe_grads* g;
    uint8_t* ws;
    WsLayout layout;
    uint32_t* err;
    uint64_t wait_ns;
};
// Rows of the padded row space the backward allocates.
int64_t bwd_padded_rows(const Dims& D);
cudaError_t launch_backward(const Dims& D, const BwdArgs& a, cudaStream_t s);

// ---- device properties, cached per device
int num_sms();

// Programmatic stream serialization (see griddep_wait) pays off only when the
// layer's kernels are short: measured on B200, it saved ~2 us of a 106 us
// single-token decode layer and cost ~10 us of a 490 us 4096-token layer —
// and as much when only the routing, permutation and schedule kernels take it
// (471 -> 481 us; the 8192-token capped layer 109.7 -> 112.3 us). So it is
// used for batches of at most kPdlMaxTokens tokens.
constexpr int kPdlMaxTokens = 64;
inline bool use_pdl(int64_t T) { return T <= kPdlMaxTokens; }

// Launch; with pdl the kernel may be scheduled before its predecessor on the
// stream completes (every kernel calls griddep_wait before touching memory).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---- optional per-kernel event timing (moe_profile_enable); no-op when off
class ProfScope {
  public:
    ProfScope(int kernel_id, cudaStream_t s);
    ~ProfScope();
    ProfScope(const ProfScope&) = delete;
    ProfScope& operator=(const ProfScope&) = delete;

  private:
    int id_;
    cudaStream_t s_;
    void* a_;
};

}  // namespace moe

// noalloc.cu — moe_permute_noalloc: the permutation (histogram, scan,
// scatter, capacity drop) with its scratch in a fixed device array of this
// library instead of a caller-provided workspace.
//
// Who needs it: code that must not call cudaMalloc (or any allocator) at the
// point where it permutes — for example a serving engine that has handed all
// free device memory to its own budget and forbids allocations afterwards, or
// a runtime without an allocator object of its own — and that still wants
// this library's permutation. Such a caller passes only its inputs and
// outputs; the per-block histograms and bases live in g_perm_scratch below.
//
// Costs and limits: the array is 128 permutation blocks x 256 experts x 2 int32
// (256 KiB) and stays allocated on every GPU that loads the
// library until the process exits. Every call uses the same array, so calls
// whose work overlaps on the GPU (different streams, or different host
// threads) race and must not be issued; calls on one stream are ordered and
// safe. The array needs no clearing between calls: each call writes every
// entry it later reads before reading it.
#include <mutex>

#include "internal.h"

namespace moe {

namespace {

// the most blocks a call may use: small batches' blocks at kPermSmallPairs, or large ones'
constexpr int kNoAllocMaxBlocks =
    (kPermSmallPairs / (kPermWarps * 32 * kPermRoundsSmall)) > (MOE_NOALLOC_MAX_PAIRS / kPermMaxPairsPerBlock)
        ? int(kPermSmallPairs / (kPermWarps * 32 * kPermRoundsSmall))
        : int(MOE_NOALLOC_MAX_PAIRS / kPermMaxPairsPerBlock);  // 128
constexpr int kNoAllocInts = 2 * kNoAllocMaxBlocks * kMaxE;                   // counts + bases

static_assert(MOE_NOALLOC_MAX_PAIRS % kPermMaxPairsPerBlock == 0, "pair limit must be whole blocks");

// The fixed scratch: per-block expert counts, then per-block expert bases.
static __device__ __align__(256) int32_t g_perm_scratch[kNoAllocInts];

// Device address of g_perm_scratch on each device, looked up once per device
// (with that device current) on the first call made there. The cached address
// belongs to that device's primary context: after cudaDeviceReset (or anything
// else that destroys the context) it is stale, so the entry point must not be
// used across a reset.
std::mutex g_mu;
int32_t* g_scratch_addr[64] = {nullptr};

int32_t* scratch_for_current_device(cudaError_t* err) {
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= 64) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> g(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_perm_scratch);
        if (*err != cudaSuccess) return nullptr;
        g_scratch_addr[dev] = static_cast<int32_t*>(p);
    }
    return g_scratch_addr[dev];
}

}  // namespace

}  // namespace moe

extern "C" MOE_API int moe_permute_noalloc(const moe_params* p, const int32_t* topk_idx, int32_t* counts,
                                           int32_t* kept_counts, int32_t* offsets, int32_t* sorted_token,
                                           int32_t* sorted_pair, int32_t* pair_row, uint32_t* err_word,
                                           moe_stream_t stream) {
    using namespace moe;
    // the same parameter checks and dimensions as moe_permute, status unchanged
    Dims D{};
    const int st = make_dims(p, &D);
    if (st != MOE_OK) return st;
    if (D.pairs > MOE_NOALLOC_MAX_PAIRS || D.perm_blocks > kNoAllocMaxBlocks)
        return MOE_ERR_WORKSPACE_TOO_SMALL;  // beyond the fixed scratch
    if (!topk_idx || !counts || !kept_counts || !offsets || !sorted_token || !sorted_pair || !pair_row ||
        !err_word)
        return MOE_ERR_INVALID_ARG;
    cudaError_t ce = cudaSuccess;
    int32_t* scratch = scratch_for_current_device(&ce);
    if (!scratch) return MOE_ERR_CUDA;
    int32_t* blockcounts = scratch;
    int32_t* blockbase = scratch + kNoAllocMaxBlocks * kMaxE;
    const cudaError_t e = launch_permute(D, topk_idx, blockcounts, blockbase, counts, kept_counts, offsets,
                                         sorted_token, sorted_pair, pair_row, err_word, stream);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

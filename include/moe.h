/*
 * moe.h — C ABI of the routed mixture-of-experts expert FFN for NVIDIA B200 (sm_100a).
 *
 * The layer: top-k routing from router logits with an optional capacity drop,
 * the token→expert permutation, per-expert gate/up GEMMs with a clamped SwiGLU,
 * the down GEMM, and the gate-weighted combine back to token order. Sources
 * (web pages, cited by title and part):
 *   - "mini-AGI PR #3" minagi/pool.py, requested(): router softmax, top-k,
 *     renormalised weights; flatten / argsort by expert / bincount; the
 *     capacity drop (keep mask, counts.clamp(max=limit)).
 *   - "mini-AGI PR #3/#4" configs/strix_halo_large.yaml, capacity_factor:
 *     the most of a batch one expert may take as a multiple of its fair
 *     share; the rest is dropped; 0 removes the cap.
 *   - "mini-AGI PR #4" minagi/pool.py, experts()/run(): silu(x W1) * (x W3),
 *     then W2; outputs read back in pair order.
 *   - "Strata PR #4366" (DS4_FAT_ROWS), Approach: clamped SwiGLU; an
 *     expert's weights decoded once, its rows gathered, one GEMM.
 *   - "TensorFold PR #1607", What this changes: served plans with an always-on
 *     shared expert ("256 + shared").
 *
 * Conventions for every call
 *   - Pointers are DEVICE pointers owned by the caller unless a parameter says
 *     "host". The library allocates no device memory: scratch comes from the
 *     caller's workspace `ws` of at least moe_workspace_size() bytes, 256-byte
 *     aligned. bf16 tensors are passed as uint16_t bit patterns.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). They make no host synchronisation, except
 *     moe_get_error() and moe_forward_host(), which say so.
 *   - Return value: MOE_OK, or an error detected on the host before any launch
 *     (nothing was launched), or MOE_ERR_CUDA if a launch failed.
 *   - Errors found on the device (a bound-checked index out of range, a
 *     bounded wait that gave up) set bits in a sticky error word at the start
 *     of the workspace; read it with moe_get_error(), reset with
 *     moe_clear_error(). A kernel that sets it stops early and returns; its
 *     outputs are then undefined.
 *   - Limits: 1 <= k <= min(E, 8); 1 <= E <= 256; d_model and d_ff multiples
 *     of 64; 0 <= T (0: empty batch); shared expert only with bf16 weights and d_ff_shared ==
 *     d_ff. Pointers to bf16/Q4G32 tensors 16-byte aligned.
 *   - Calls that share one workspace must not overlap on the GPU.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* same object as cudaStream_t */

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* return codes */
#define MOE_OK                      0
#define MOE_ERR_INVALID_ARG         1 /* a size or flag outside the limits above */
#define MOE_ERR_WORKSPACE_TOO_SMALL 2
#define MOE_ERR_UNSUPPORTED         3 /* valid, but not implemented (see limits) */
#define MOE_ERR_CUDA                4 /* a CUDA call or launch failed */
#define MOE_ERR_MISALIGNED          5 /* a pointer without the 16-byte alignment */
#define MOE_ERR_DEVICE              6 /* moe_get_error: the device error word is set */

/* device error word bits (moe_get_error) */
#define MOE_DEVERR_TIMEOUT 0x1u /* a bounded wait in a pipelined kernel gave up */
#define MOE_DEVERR_BOUNDS  0x2u /* an expert id or row index outside its range */
#define MOE_DEVERR_RANGE   0x4u /* an fp16 intermediate (h or y) beyond +-65504 or NaN */

/* weight formats */
#define MOE_WEIGHTS_BF16  0
#define MOE_WEIGHTS_Q4G32 1

/* expert kernel variants */
#define MOE_VARIANT_AUTO   0 /* per expert, from its kept rows (stream_max_rows) */
#define MOE_VARIANT_TENSOR 1 /* every expert on the tcgen05 tile kernels */
#define MOE_VARIANT_STREAM 2 /* every expert on the few-rows weight-streaming kernels */

/* layer output dtype */
#define MOE_OUT_F32  0 /* fp32 (default): the residual stream's dtype */
#define MOE_OUT_BF16 1

/* dtype of w_down / shared_down (bf16 weight format only) */
#define MOE_DOWN_BF16 0 /* as given; each tile is converted to fp16 in shared memory */
#define MOE_DOWN_F16  1 /* prepared once with moe_convert_bf16_to_f16 (load time) */

/* SMs per tcgen05 tile (moe_params.tile_ctas) */
#define MOE_TILE_AUTO 0 /* library default: MOE_TILE_ONE (moe_tile_ctas tells which) */
#define MOE_TILE_ONE  1 /* one SM per 128-row x 256-column tile */
#define MOE_TILE_PAIR 2 /* two SMs (a cluster, tcgen05 cta_group::2) per 256-row x 256-column
                           tile, for the bf16 gate/up and the fp16 down GEMMs; a third less
                           L2-to-SM traffic per FLOP, at the price of rounding each expert's
                           rows up to 256. Down with W_down given as bf16 and all Q4G32 GEMMs
                           keep one SM per tile. Measured on B200 slower than MOE_TILE_ONE on
                           the 4096-token prompt layer, so it is opt-in. */

/* workspace kinds for moe_workspace_size() */
#define MOE_WS_ROUTE        0
#define MOE_WS_PERMUTE      1
#define MOE_WS_EXPERT_FFN   2
#define MOE_WS_COMBINE      3
#define MOE_WS_FORWARD      4
#define MOE_WS_FORWARD_HOST 5
#define MOE_WS_ROUTE_STATS  6
#define MOE_WS_BACKWARD     7

typedef struct moe_params {
    int32_t T;               /* tokens in this call; 0 = empty batch: every call returns MOE_OK
                                without a kernel launch (buffers may then be null); moe_permute
                                and moe_forward's counts_out get zero counts and offsets */
    int32_t d_model;         /* d */
    int32_t d_ff;            /* f, per routed expert */
    int32_t E;               /* routed experts */
    int32_t k;               /* experts per token */
    float capacity_factor;   /* 0 = no cap; else cap = ceil(cf * T * k / E) rows per expert,
                                computed in double from this float */
    float swiglu_limit;      /* L: gate and up pre-activations are clamped to [-L, L]; <= 0: no clamp */
    int32_t weight_format;   /* MOE_WEIGHTS_* for the routed experts */
    int32_t has_shared;      /* 1: add an always-on, un-gated shared expert */
    int32_t d_ff_shared;     /* its f (must equal d_ff) */
    int32_t variant;         /* MOE_VARIANT_* */
    int32_t stream_max_rows; /* AUTO: experts with 1..this many kept rows use the streaming
                                kernels, the rest the tcgen05 tiles; < 0 = library default
                                from the measured table (moe_variant_table) */
    int32_t out_dtype;       /* MOE_OUT_F32 | MOE_OUT_BF16 */
    int32_t down_dtype;      /* MOE_DOWN_BF16 | MOE_DOWN_F16 */
    int32_t tile_ctas;       /* SMs per tcgen05 tile: MOE_TILE_* */
} moe_params;

/*
 * Expert weights (device pointers).
 *   BF16:  w_gate, w_up [E, d, f]; w_down [E, f, d]; row-major bf16; s_* NULL.
 *   Q4G32 (self-defined): a matrix of reduction length K and output width N
 *          is stored K-major as packed bytes [N, K/2]: each row is K/8
 *          little-endian 32-bit words; word i holds k = 8i..8i+7, nibble
 *          position p (bits 4p..4p+3) holding k = 8i + {0,2,4,6,1,3,5,7}[p];
 *          each nibble u = q + 8, q in [-7, 7]. Scales are fp16, group-major
 *          [K/32, N]: one per group of 32 consecutive k of a column. The
 *          weight is q * s.
 *          w_gate, w_up: [E, f, d/2] bytes, s_gate, s_up: [E, d/32, f] fp16;
 *          w_down: [E, d, f/2] bytes, s_down: [E, f/32, d] fp16.
 *   shared_*: bf16 [d, f], [d, f], [f, d] of the shared expert; NULL if has_shared = 0.
 */
typedef struct moe_weights {
    const void* w_gate;
    const void* w_up;
    const void* w_down;
    const void* s_gate;
    const void* s_up;
    const void* s_down;
    const void* shared_gate;
    const void* shared_up;
    const void* shared_down;
} moe_weights;

/* Library version (major*10000 + minor*100 + patch). */
MOE_API int moe_version(void);

/* Human-readable name of a return code. */
MOE_API const char* moe_status_string(int status);

/*
 * Per-expert capacity: *cap = ceil(cf * T * k / E), or -1 when cf <= 0.
 * ("mini-AGI" capacity_factor; see the file comment.)
 */
MOE_API int moe_capacity(const moe_params* p, int32_t* cap);

/*
 * Rows of the permuted buffers (sorted_token, sorted_pair, y_rows):
 * min(T*k, E*cap) (T*k with no cap) plus T when has_shared.
 */
MOE_API int moe_max_rows(const moe_params* p, int64_t* rows);

/*
 * SMs per tcgen05 tile that calls with these params use for the bf16 gate/up
 * GEMM (MOE_TILE_ONE or MOE_TILE_PAIR), into *ctas. MOE_TILE_AUTO resolves to
 * MOE_TILE_ONE; MOE_TILE_PAIR with Q4G32 weights resolves to MOE_TILE_ONE.
 */
MOE_API int moe_tile_ctas(const moe_params* p, int32_t* ctas);

/*
 * The measured table behind the default variant choice (stream_max_rows < 0):
 * row i says that experts of at most max_rows[i] kept rows take the weight-
 * streaming kernels while the touched experts' gate/up tiles (min(E', T*k +
 * has_shared) experts x ceil(d_ff/128)) number fewer than tiles_per_sm[i] x
 * the GPU's SMs; the first matching row applies, and past the last every
 * expert takes the tcgen05 tiles. The pages' analogues are Strata PR #4366's
 * light kernels for experts of <= 16 rows and TensorFold PR #1607's bound on
 * pairs per item ("What this changes"); these entries were measured on B200.
 * Copies up to n rows into the host arrays; returns the table's row count.
 */
MOE_API int moe_variant_table(float* tiles_per_sm, int32_t* max_rows, int n);

/* Bytes of workspace each call needs (which = MOE_WS_*); 0 on invalid params. */
MOE_API size_t moe_workspace_size(const moe_params* p, int which);

/*
 * moe_route — S1 of the path: per token, the top-k experts and their weights.
 *   "mini-AGI PR #3" requested(): softmax of the logits, top-k, renormalised
 *   (= a softmax over the k selected logits).
 * logits   fp32 [T, E] row-major (finite; NaN is outside the contract).
 * topk_idx int32 [T, k]: expert ids in descending logit order; equal logits
 *          go to the lower index (-0.0 equals +0.0). Compared exactly in fp32.
 * topk_w   fp32 [T, k]: exp(l_j - l_max) / sum over the k selected.
 */
MOE_API int moe_route(const moe_params* p, const float* logits, int32_t* topk_idx, float* topk_w,
              void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_route_stats — moe_route plus the router's telemetry, in the same kernel.
 *   "mini-AGI PR #3" requested(), telemetry hunk, on the full softmax p of
 *   each token's logits (p[t, e] = exp(l - lse)):
 *   stats[0] kept     mean over tokens of the top-k mass sum_j p[t, idx[t, j]],
 *                     measured before the weights are renormalised
 *   stats[1] want_k   mean over tokens of the fewest experts, largest p first
 *                     (ties to the lower index), whose p sum to at least 0.9
 *   stats[2] balance  E * sum_e frac[e] * mean_t p[t, e], frac[e] = share of
 *                     tokens whose first choice idx[t, 0] is e
 *   stats[3] z        mean over tokens of logsumexp(logits[t])^2
 *   stats[4] aux      balance + z_weight * z (the page's default weight: 1e-3)
 *   The page's running averages across calls (pressure = EMA of 1 - kept,
 *   want_k = EMA of want) are the caller's state; these are per-batch values.
 * topk_idx, topk_w  as moe_route (bit-identical to it).
 * stats         device fp32 [5] (required).
 * kept_tok      device fp32 [T] per-token top-k mass, or NULL.
 * want_tok      device int32 [T] per-token count, or NULL.
 * expert_stats  device fp32 [2, E]: frac, then mean p per expert; or NULL.
 * ws: MOE_WS_ROUTE_STATS bytes (per-block partial sums). Deterministic: fixed
 * summation orders (fp32 within a block of tokens, fp64 across blocks). With
 * T = 0 nothing is launched and stats is not written.
 */
MOE_API int moe_route_stats(const moe_params* p, const float* logits, int32_t* topk_idx, float* topk_w,
              float z_weight, float* stats, float* kept_tok, int32_t* want_tok, float* expert_stats,
              void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_permute — S2/S3: histogram, prefix offsets, scatter, capacity drop.
 *   "mini-AGI PR #3" requested(): pairs sorted by expert, bincount, the keep
 *   mask over each expert's pairs, counts clamped to the limit.
 * Pair p = t*k + j. Let E' = E + has_shared.
 * topk_idx     int32 [T, k] (ids in [0, E); out-of-range ids set MOE_DEVERR_BOUNDS)
 * counts       int32 [E']   pairs requested per expert (shared: T)
 * kept_counts  int32 [E']   min(counts, cap)
 * offsets      int32 [E'+1] exclusive prefix of kept_counts; offsets[E'] = rows used
 * sorted_token int32 [moe_max_rows] token of each row; within an expert ascending
 * sorted_pair  int32 [moe_max_rows] pair of each row (-1 for shared rows)
 * pair_row     int32 [T*k]  row of each pair, -1 if dropped
 * The drop keeps, per expert, its first cap pairs in token order. Bit-exact:
 * the result is unique (no atomics decide an order).
 */
MOE_API int moe_permute(const moe_params* p, const int32_t* topk_idx, int32_t* counts,
                int32_t* kept_counts, int32_t* offsets, int32_t* sorted_token,
                int32_t* sorted_pair, int32_t* pair_row, void* ws, size_t ws_bytes,
                moe_stream_t stream);

/*
 * moe_permute_noalloc — moe_permute without a workspace argument. The pages
 * have no counterpart: this is a library convenience, not a step of the method.
 * It computes exactly what moe_permute computes (same outputs, same layouts,
 * bit-identical) but keeps its scratch (per-block histograms and bases) in a
 * fixed array inside the library, so the caller passes only inputs, outputs
 * and a device error word.
 * Who needs it: callers that must not allocate device memory when they
 * permute — an engine that has already handed all free memory to its own
 * budget, or a plugin without an allocator of its own.
 * Limit: T*k <= MOE_NOALLOC_MAX_PAIRS; larger calls return
 * MOE_ERR_WORKSPACE_TOO_SMALL before any launch (use moe_permute). The array
 * (256 KiB) stays resident on every GPU that loads the library until exit.
 * err_word  device uint32, OR-ed with MOE_DEVERR_BOUNDS for out-of-range ids
 *           (the caller zeroes it; it is not cleared here).
 * Returns the status moe_permute returns for the same parameters (one shared
 * check), and MOE_ERR_INVALID_ARG for null pointers. The first call on a
 * device looks up the array's device address (a CUDA runtime query, no
 * allocation) and keeps it for the life of the process: make that first call
 * before any stream capture, and do not use this entry point across a
 * cudaDeviceReset (the kept address would be stale). Every call uses the same array, so calls whose work may
 * overlap on the GPU (other streams, other host threads) race: issue them on
 * one stream. Nothing here calls an allocator.
 */
#define MOE_NOALLOC_MAX_PAIRS 262144
MOE_API int moe_permute_noalloc(const moe_params* p, const int32_t* topk_idx, int32_t* counts,
                int32_t* kept_counts, int32_t* offsets, int32_t* sorted_token,
                int32_t* sorted_pair, int32_t* pair_row, uint32_t* err_word,
                moe_stream_t stream);

/*
 * moe_expert_ffn — S4..S6 (+ S8, S9): per expert e, rows r in
 * [offsets[e], offsets[e+1]):
 *   g = x[sorted_token[r]] W_gate[e],  u = x[sorted_token[r]] W_up[e]
 *   h = silu(clamp(g, -L, L)) * clamp(u, -L, L)        (fp32, then fp16)
 *   y_rows[r] = w_r * (h W_down[e])                     (fp32, then fp16)
 * with w_r = topk_w[sorted_pair[r]] (1 for shared rows).
 *   "mini-AGI PR #4" experts(); "Strata PR #4366" Approach (clamped SwiGLU,
 *   an expert's weights decoded once and its rows gathered).
 * x       bf16 [T, d]; offsets / sorted_token / sorted_pair as moe_permute writes them
 * topk_w  fp32 [T, k]
 * y_rows  fp16 [moe_max_rows, d]; rows past offsets[E'] are not written.
 * Precision: x and the gate/up weights enter the tensor cores as given (bf16),
 * fp32 accumulate; h is kept in fp16 and the down GEMM runs in fp16 (each
 * W_down tile is converted bf16 -> fp16 in shared memory, exact for values in
 * fp16's normal range), fp32 accumulate; y in fp16. A value of h or y past
 * +-65504 sets MOE_DEVERR_RANGE. (Strata PR #4366 runs its expert GEMM and
 * SwiGLU in FP16 for the same reason: more significand than bf16.)
 * Each expert runs either the tcgen05 tile kernels or the few-rows streaming
 * kernels (params.variant / stream_max_rows). Weights of experts without rows
 * are never read.
 */
MOE_API int moe_expert_ffn(const moe_params* p, const uint16_t* x, const int32_t* offsets,
                   const int32_t* sorted_token, const int32_t* sorted_pair,
                   const float* topk_w, const moe_weights* w, uint16_t* y_rows,
                   void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_combine — S7: out[t] = sum over j in 0..k-1 with pair_row[t*k+j] >= 0 of
 * y_rows[pair_row[t*k+j]] (fp16, already gate-weighted), plus y_rows[offsets[E] + t]
 * when has_shared; fp32 in fixed j order, written as out_dtype (fp32 by
 * default, or bf16). Deterministic.
 *   "mini-AGI PR #4" run(): outputs gathered back in pair order and summed.
 * A dropped pair adds nothing; the other weights are not renormalised.
 * offsets may be NULL when has_shared = 0.
 */
MOE_API int moe_combine(const moe_params* p, const uint16_t* y_rows, const int32_t* pair_row,
                const int32_t* offsets, void* out, void* ws, size_t ws_bytes,
                moe_stream_t stream);

/*
 * moe_forward — the whole layer (route → permute → expert FFN → combine) on
 * one stream with no host synchronisation; intermediates live in ws.
 * x bf16 [T, d], logits fp32 [T, E], out [T, d] of out_dtype (fp32 default).
 * counts_out: NULL, or int32 [E'] receiving the per-expert requested counts.
 */
MOE_API int moe_forward(const moe_params* p, const uint16_t* x, const float* logits,
                const moe_weights* w, void* out, int32_t* counts_out,
                void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_forward_host — moe_forward with HOST x, logits and out (weights stay on
 * the device): copies x and logits in, runs the layer, copies out back, then
 * synchronises the stream. Host buffers may be pageable; pinned is faster.
 * ws: MOE_WS_FORWARD_HOST bytes (holds device copies of x, logits, out).
 */
MOE_API int moe_forward_host(const moe_params* p, const uint16_t* x_host, const float* logits_host,
                     const moe_weights* w, void* out_host, void* ws, size_t ws_bytes,
                     moe_stream_t stream);

/*
 * moe_forward_host_async — moe_forward_host without the final synchronisation:
 * the copies in, the layer and the copy out are enqueued on `stream` and the
 * call returns. The caller synchronises the stream (or an event recorded on it)
 * before it reads out_host or writes x_host / logits_host again. With pinned
 * host buffers the copies run asynchronously, so calls on two streams with
 * separate workspaces and buffers overlap one step's copies with another's
 * kernels (a pipelined serving loop); pageable buffers make the copies
 * synchronous with the host. Same arguments and errors as moe_forward_host.
 */
MOE_API int moe_forward_host_async(const moe_params* p, const uint16_t* x_host, const float* logits_host,
                     const moe_weights* w, void* out_host, void* ws, size_t ws_bytes,
                     moe_stream_t stream);

/*
 * Weight preparation, done once at load time, outside the layer's calls:
 * dst[i] = fp16(src[i]) for n bf16 values (round to nearest even; exact for
 * |v| in fp16's normal range and for bf16 values down to 2^-17). Used to keep
 * an fp16 copy of W_down so the down GEMM reads fp16 directly (down_dtype =
 * MOE_DOWN_F16): the layer keeps h in fp16 for precision, and one tcgen05 MMA
 * takes a single operand type. Values beyond +-65504 set bit MOE_DEVERR_RANGE
 * in *err_ws's error word when err_ws is not NULL. Asynchronous.
 */
MOE_API int moe_convert_bf16_to_f16(const uint16_t* src, uint16_t* dst, int64_t n, void* err_ws,
                                    moe_stream_t stream);

/*
 * Synchronises `stream`, then reads the sticky device error word at the start
 * of ws into *err (host). Returns MOE_OK if it is 0, MOE_ERR_DEVICE if not.
 */
MOE_API int moe_get_error(const void* ws, uint32_t* err, moe_stream_t stream);

/* Resets the device error word (asynchronous). */
MOE_API int moe_clear_error(void* ws, moe_stream_t stream);

/*
 * Test hook: the time limit, in nanoseconds, of every bounded wait in the
 * pipelined kernels launched after this call by this process (default 1 s).
 * 0 restores the default.
 */
MOE_API int moe_set_wait_limit_ns(uint64_t ns);

/*
 * Self-test of the failure path (the pages have no counterpart): one tiny
 * kernel waits, with the same bounded wait as the pipelined kernels, on an
 * mbarrier that nothing completes. After limit_ns (1 .. 1e10) it gives up,
 * ORs MOE_DEVERR_TIMEOUT into the error word at err_ws and returns, so the
 * context stays usable. Asynchronous; read the word with moe_get_error().
 */
MOE_API int moe_wait_selftest(void* err_ws, uint64_t limit_ns, moe_stream_t stream);

/*
 * Kernel ids for the profiler and moe_launch_count(). Each is one kernel of
 * the library; a call launches a fixed sequence of them (no host sync).
 */
#define MOE_K_ROUTE          0  /* S1 top-k softmax router */
#define MOE_K_PERM_COUNT     1  /* S2 per-block histograms */
#define MOE_K_PERM_SCAN      2  /* S2 block bases, counts, kept, offsets */
#define MOE_K_PERM_SCATTER   3  /* S3 ranks, drop, row lists (in moe_forward also the
                                   scan's outputs and the schedule, when they fit) */
#define MOE_K_SCHEDULE       4  /* per-expert variant choice and M-tile prefix */
#define MOE_K_GATHER         5  /* S4 row gather for the tile kernels */
#define MOE_K_TC_GATEUP      6  /* S5 tcgen05 gate/up GEMM + clamped SwiGLU */
#define MOE_K_TC_DOWN        7  /* S6 tcgen05 down GEMM + gate scale */
#define MOE_K_STREAM_GATEUP  8  /* S8 few-rows gate/up (weight streaming) */
#define MOE_K_STREAM_REDUCE  9  /* S8 K-split partial sums + SwiGLU */
#define MOE_K_STREAM_DOWN   10  /* S8 few-rows down */
#define MOE_K_COMBINE       11  /* S7 gate-weighted combine */
#define MOE_K_CONVERT       12  /* load-time bf16 -> fp16 weight copy (not a layer step) */
#define MOE_K_FRONT         13  /* S1-S3 + schedule fused, moe_forward with T <= 64 */
#define MOE_K_ROUTE_STATS   14  /* router telemetry: the final sum over blocks (moe_route_stats) */
#define MOE_K_BWD_GEMM      15  /* backward tcgen05 GEMMs (moe_expert_ffn_backward) */
#define MOE_K_BWD_SMALL     16  /* backward schedule, gathers, zeroing, reductions */
#define MOE_K_COUNT         17

/*
 * Gradients written by moe_expert_ffn_backward (device pointers, fp32, row-major).
 *   dx           [T, d]      required
 *   dw_gate      [E, d, f]   required (experts without rows get zeros)
 *   dw_up        [E, d, f]   required
 *   dw_down      [E, f, d]   required
 *   d_topk_w     [T, k]      required: dL / d topk_w (0 for a dropped pair)
 *   dlogits      [T, E]      or NULL: through the softmax over the k selected
 *                            logits (0 off the selected experts); needs topk_idx
 *   dshared_*    [d, f], [d, f], [f, d] with has_shared, else NULL
 */
typedef struct moe_grads {
    float* dx;
    float* dw_gate;
    float* dw_up;
    float* dw_down;
    float* d_topk_w;
    float* dlogits;
    float* dshared_gate;
    float* dshared_up;
    float* dshared_down;
} moe_grads;

/*
 * moe_expert_ffn_backward — gradients of the layer (S5-S7 and the routing
 * weights) for an upstream gradient dout = dL/d out.
 *   "mini-AGI PR #3" tests/test_dispatch.py: the layer trains through this
 *   path and the expert weights (w1, w3, w2 = gate, up, down) get the same
 *   gradients on every dispatch path. With y = swiglu(x Wg, x Wu) Wd and
 *   out[t] = sum_j w[t,j] y[t,j] (+ shared): a kept pair's expert sees
 *   dy = w dout[t]; dh = dy Wd^T; dg, du from the clamped SwiGLU (the clamp
 *   passes the gradient where -L <= v <= L); dx = sum over the token's pairs
 *   of dg Wg^T + du Wu^T; dWd = h^T dy, dWg = x^T dg, dWu = x^T du over each
 *   expert's rows; d w[t,j] = <dout[t], y[t,j]>; dlogits_j = w_j (dw_j -
 *   sum_i w_i dw_i).
 * Inputs are the forward's: x bf16 [T, d]; topk_idx, topk_w (moe_route);
 * offsets, sorted_token, sorted_pair, pair_row (moe_permute); weights as for
 * moe_forward with down_dtype MOE_DOWN_F16: bf16 W_gate, W_up and the fp16
 * copy of W_down (and of the shared expert's) that moe_convert_bf16_to_f16
 * prepares; dout fp32 [T, d]. g: see moe_grads.
 * Arithmetic on the tcgen05 tensor cores with fp32 accumulation: g and u are
 * recomputed in fp32; products with the bf16 gate/up weights take bf16
 * operands (x; dg, du rounded once), the product with W_down and the weight
 * gradients take fp16 operands (dout rows, h, dg, du rounded once).
 * ws: MOE_WS_BACKWARD bytes. Returns MOE_ERR_UNSUPPORTED for Q4G32 weights or
 * a bf16 W_down. Deterministic (no atomics decide a sum).
 */
MOE_API int moe_expert_ffn_backward(const moe_params* p, const uint16_t* x, const int32_t* topk_idx,
              const float* topk_w, const int32_t* offsets, const int32_t* sorted_token,
              const int32_t* sorted_pair, const int32_t* pair_row, const moe_weights* w,
              const float* dout, const moe_grads* g, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Number of kernel launches one call of `which` (MOE_WS_ROUTE .. MOE_WS_BACKWARD,
 * naming moe_route .. moe_forward_host, moe_route_stats, moe_expert_ffn_backward)
 * makes with these params, into *n (host). For moe_expert_ffn_backward the count
 * includes the routing-logit gradient, launched when dlogits is given (one fewer
 * without).
 */
MOE_API int moe_launch_count(const moe_params* p, int which, int* n);

/*
 * Per-kernel timing. moe_profile_enable(1): from then on every launch is
 * bracketed by two CUDA events recorded on its stream (cheap; off by default).
 * moe_profile_collect(): waits for the recorded events, writes the summed
 * milliseconds and launch counts per kernel id (host arrays of MOE_K_COUNT)
 * and forgets them.
 */
MOE_API int moe_profile_enable(int on);
MOE_API int moe_profile_collect(double* total_ms, int64_t* launches);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */

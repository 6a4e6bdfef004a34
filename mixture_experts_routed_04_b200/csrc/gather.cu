// gather.cu — S4: the row gather. xg[r] = x[sorted_token[r]] for every row
// of every expert, in expert order, so the GEMMs' A operand (and the streaming
// kernels' rows tile) is a plain TMA box. A gather inside the GEMM (TMA
// tile::gather4, or cp.async warps: gemm_tc.cu's GATHER kernels) was measured
// slower on B200.
#include "internal.h"

namespace moe {

// xg[r] = x[sorted_token[r]] for r < offsets[Etot]. One warp per row (grid
// stride): the row's token is read once, then each lane moves up to eight
// 16-byte vectors of the row with all its loads in flight before its stores.
// TO_F16: bf16 -> fp16 on the way (the Q4G32 path runs its MMAs in fp16).
template <bool TO_F16>
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x,
                                                          const int32_t* __restrict__ sorted_token,
                                                          const int32_t* __restrict__ offsets, int Etot, int d,
                                                          int T, uint16_t* __restrict__ xg, uint32_t* err) {
    griddep_wait();
    griddep_launch();
    const int lane = threadIdx.x & 31;
    const int vec = d / 8;
    const int64_t rows = offsets[Etot];
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const int t = __ldg(sorted_token + r);
        if (t < 0 || t >= T) {
            if (lane == 0) set_error(err, MOE_DEVERR_BOUNDS);
            continue;
        }
        const uint4* src = reinterpret_cast<const uint4*>(x + int64_t(t) * d);
        uint4* dst = reinterpret_cast<uint4*>(xg + r * d);
        for (int c0 = 0; c0 < vec; c0 += 8 * 32) {
            uint4 v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c = c0 + i * 32 + lane;
                if (c < vec) v[i] = __ldg(src + c);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c = c0 + i * 32 + lane;
                if (c < vec) {
                    if (TO_F16) {
                        v[i].x = bf16x2_to_f16x2(v[i].x);
                        v[i].y = bf16x2_to_f16x2(v[i].y);
                        v[i].z = bf16x2_to_f16x2(v[i].z);
                        v[i].w = bf16x2_to_f16x2(v[i].w);
                    }
                    dst[c] = v[i];
                }
            }
        }
    }
}

// The same rows in token order, for moe_forward, which has pair_row: one warp
// per token reads x[t] once and writes it to each of the token's kept rows
// (pair_row[t*k + j] >= 0) and, with a shared expert, to row offsets[E] + t.
// x is read once instead of k times (at T = 32768, d = 2048 it exceeds L2).
template <bool TO_F16>
__global__ void __launch_bounds__(256) scatter_rows_kernel(const uint16_t* __restrict__ x,
                                                           const int32_t* __restrict__ pair_row,
                                                           const int32_t* __restrict__ offsets, int T, int k, int E,
                                                           int has_shared, int d, int64_t rows,
                                                           uint16_t* __restrict__ xg, uint32_t* err) {
    griddep_wait();
    griddep_launch();
    const int lane = threadIdx.x & 31;
    const int vec = d / 8;
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
    const int shared_row0 = has_shared ? offsets[E] : 0;
    for (int64_t t = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
        int r = lane < k ? pair_row[t * k + lane] : -1;
        if (r >= rows) {
            set_error(err, MOE_DEVERR_BOUNDS);
            r = -1;
        }
        int dst[kMaxK + 1];
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) dst[j] = __shfl_sync(0xFFFFFFFFu, r, j);
        dst[kMaxK] = has_shared ? shared_row0 + int(t) : -1;
        const uint4* src = reinterpret_cast<const uint4*>(x + t * d);
        for (int c = lane; c < vec; c += 32) {
            uint4 v = __ldg(src + c);
            if (TO_F16) {
                v.x = bf16x2_to_f16x2(v.x);
                v.y = bf16x2_to_f16x2(v.y);
                v.z = bf16x2_to_f16x2(v.z);
                v.w = bf16x2_to_f16x2(v.w);
            }
#pragma unroll
            for (int j = 0; j <= kMaxK; ++j)
                if (dst[j] >= 0) reinterpret_cast<uint4*>(xg + int64_t(dst[j]) * d)[c] = v;
        }
    }
}

cudaError_t launch_scatter_rows(const Dims& D, const uint16_t* x, const int32_t* pair_row, const int32_t* offsets,
                                uint16_t* xg, uint32_t* err, cudaStream_t s) {
    int64_t blocks = (int64_t(D.T) + 7) / 8;  // 8 warps (tokens) per block
    const int64_t cap = int64_t(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    {
        ProfScope prof_(MOE_K_GATHER, s);
        const bool pdl = use_pdl(D.T);
        const cudaError_t le =
            D.fmt == MOE_WEIGHTS_Q4G32
                ? launch_pdl(pdl, scatter_rows_kernel<true>, dim3(int(blocks)), dim3(256), 0, s, x, pair_row,
                             offsets, D.T, D.k, D.E, D.has_shared, D.d, int64_t(D.rows), xg, err)
                : launch_pdl(pdl, scatter_rows_kernel<false>, dim3(int(blocks)), dim3(256), 0, s, x, pair_row,
                             offsets, D.T, D.k, D.E, D.has_shared, D.d, int64_t(D.rows), xg, err);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

cudaError_t launch_gather(const Dims& D, const uint16_t* x, const int32_t* sorted_token, const int32_t* offsets,
                          uint16_t* xg, uint32_t* err, cudaStream_t s) {
    int64_t blocks = (D.rows + 7) / 8;  // 8 warps (rows) per block
    const int64_t cap = int64_t(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    {
        ProfScope prof_(MOE_K_GATHER, s);
        const bool pdl = use_pdl(D.T);
        const cudaError_t le =
            D.fmt == MOE_WEIGHTS_Q4G32
                ? launch_pdl(pdl, gather_rows_kernel<true>, dim3(int(blocks)), dim3(256), 0, s, x, sorted_token,
                             offsets, D.Etot, D.d, D.T, xg, err)
                : launch_pdl(pdl, gather_rows_kernel<false>, dim3(int(blocks)), dim3(256), 0, s, x, sorted_token,
                             offsets, D.Etot, D.d, D.T, xg, err);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe

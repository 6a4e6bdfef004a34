// gather.cu — S4: the row gather. xg[r] = x[sorted_token[r]] for every row
// of every expert, in expert order, so the GEMMs' A operand (and the streaming
// kernels' rows tile) is a plain TMA box. A gather inside the GEMM (TMA
// tile::gather4 or cp.async warps) was measured slower on B200, and so was a
// 4-way unrolled version of this loop.
#include "internal.h"

namespace moe {

// xg[r] = x[sorted_token[r]] for r < offsets[Etot]; 16-byte vectors. TO_F16:
// bf16 -> fp16 on the way (the Q4G32 path runs its MMAs in fp16).
template <bool TO_F16>
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x,
                                                          const int32_t* __restrict__ sorted_token,
                                                          const int32_t* __restrict__ offsets, int Etot, int d,
                                                          int T, uint16_t* __restrict__ xg, uint32_t* err) {
    griddep_wait();
    griddep_launch();
    const int vec = d / 8;
    const int64_t total = int64_t(offsets[Etot]) * vec;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = i / vec;
        const int c = int(i - r * vec);
        const int t = __ldg(sorted_token + r);
        if (t < 0 || t >= T) {
            set_error(err, MOE_DEVERR_BOUNDS);
            continue;
        }
        uint4 v = __ldg(reinterpret_cast<const uint4*>(x + int64_t(t) * d) + c);
        if (TO_F16) {
            v.x = bf16x2_to_f16x2(v.x);
            v.y = bf16x2_to_f16x2(v.y);
            v.z = bf16x2_to_f16x2(v.z);
            v.w = bf16x2_to_f16x2(v.w);
        }
        reinterpret_cast<uint4*>(xg + r * d)[c] = v;
    }
}

cudaError_t launch_gather(const Dims& D, const uint16_t* x, const int32_t* sorted_token, const int32_t* offsets,
                          uint16_t* xg, uint32_t* err, cudaStream_t s) {
    const int64_t total = D.rows * (D.d / 8);
    int64_t blocks = (total + 255) / 256;
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

// combine.cu — S7: gate-weighted outputs summed back to token order.
//
// "mini-AGI PR #4", minagi/pool.py run(): the expert outputs are read back in
// pair order (y[e_sorted, slot]) and each token's k outputs are summed with
// their gate weights. The weights were applied in the down-projection
// epilogue, so here out[t] = sum over kept j of y_rows[pair_row[t*k+j]]
// (+ the shared expert's row), accumulated in fp32 in fixed j order and
// stored as fp32 (or, with the bf16 output option, rounded to bf16 once).
// A dropped pair (row -1) adds nothing.
//
// HBM-bound: one 16-byte vector (8 bf16) per thread per row read; blocks walk
// tokens with a grid stride; no atomics, so the result is deterministic.
#include "internal.h"

namespace moe {

namespace {

template <bool OUT_BF16>
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ y_rows,
                                                      const int32_t* __restrict__ pair_row,
                                                      const int32_t* __restrict__ offsets, int T, int d, int k,
                                                      int E, int has_shared, void* __restrict__ out) {
    griddep_wait();
    griddep_launch();
    const int vec_per_row = d / 8;  // d % 64 == 0
    const int64_t total = int64_t(T) * vec_per_row;
    const int shared_base = has_shared ? offsets[E] : 0;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t t = i / vec_per_row;
        const int c = int(i - t * vec_per_row);
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        auto add = [&](const uint4& v) {
            acc[0] += f16_lo(v.x); acc[1] += f16_hi(v.x);
            acc[2] += f16_lo(v.y); acc[3] += f16_hi(v.y);
            acc[4] += f16_lo(v.z); acc[5] += f16_hi(v.z);
            acc[6] += f16_lo(v.w); acc[7] += f16_hi(v.w);
        };
        // all of the token's row loads in flight first, then the sum in the fixed order j = 0..k-1
        int rr[kMaxK];
        uint4 yv[kMaxK];
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) rr[j] = j < k ? pair_row[t * k + j] : -1;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (rr[j] >= 0) yv[j] = __ldg(reinterpret_cast<const uint4*>(y_rows + int64_t(rr[j]) * d) + c);
        uint4 ys = make_uint4(0, 0, 0, 0);
        if (has_shared) ys = __ldg(reinterpret_cast<const uint4*>(y_rows + (shared_base + t) * d) + c);
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (rr[j] >= 0) add(yv[j]);
        if (has_shared) add(ys);
        if (OUT_BF16) {
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]);
            o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]);
            o.w = pack_bf16x2(acc[6], acc[7]);
            reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + t * d)[c] = o;
        } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + t * d + c * 8);
            dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
    }
}

}  // namespace

cudaError_t launch_combine(const Dims& D, const uint16_t* y_rows, const int32_t* pair_row, const int32_t* offsets,
                           void* out, cudaStream_t s) {
    const int64_t total = int64_t(D.T) * (D.d / 8);
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    const int64_t cap = int64_t(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    {
        ProfScope prof_(MOE_K_COMBINE, s);
        const bool pdl = use_pdl(D.T);
        const cudaError_t le =
            D.out_bf16 ? launch_pdl(pdl, combine_kernel<true>, dim3(int(blocks)), dim3(threads), 0, s, y_rows,
                                    pair_row, offsets, D.T, D.d, D.k, D.E, D.has_shared, out)
                       : launch_pdl(pdl, combine_kernel<false>, dim3(int(blocks)), dim3(threads), 0, s, y_rows,
                                    pair_row, offsets, D.T, D.d, D.k, D.E, D.has_shared, out);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe

namespace moe {

namespace {

// dst = fp16(src), 8 values per thread per step; out-of-range values flagged.
__global__ void __launch_bounds__(256) convert_bf16_f16_kernel(const uint16_t* __restrict__ src,
                                                               uint16_t* __restrict__ dst, int64_t n, uint32_t* err) {
    griddep_wait();
    griddep_launch();
    bool bad = false;
    const int64_t nv = n / 8;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < nv; i += int64_t(gridDim.x) * blockDim.x) {
        uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
        bad |= !(f16_range_ok(bf16_lo(v.x)) && f16_range_ok(bf16_hi(v.x)) && f16_range_ok(bf16_lo(v.y)) &&
                 f16_range_ok(bf16_hi(v.y)) && f16_range_ok(bf16_lo(v.z)) && f16_range_ok(bf16_hi(v.z)) &&
                 f16_range_ok(bf16_lo(v.w)) && f16_range_ok(bf16_hi(v.w)));
        v.x = bf16x2_to_f16x2(v.x);
        v.y = bf16x2_to_f16x2(v.y);
        v.z = bf16x2_to_f16x2(v.z);
        v.w = bf16x2_to_f16x2(v.w);
        reinterpret_cast<uint4*>(dst)[i] = v;
    }
    for (int64_t i = nv * 8 + int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x) {
        const float f = bf16_to_f32(src[i]);
        bad |= !f16_range_ok(f);
        dst[i] = uint16_t(pack_f16x2(f, 0.f) & 0xFFFFu);
    }
    if (bad) set_error(err, MOE_DEVERR_RANGE);
}

}  // namespace

cudaError_t launch_convert_bf16_f16(const uint16_t* src, uint16_t* dst, int64_t n, uint32_t* err, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    int64_t blocks = (n / 8 + 255) / 256;
    const int64_t cap = int64_t(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    {
        ProfScope prof_(MOE_K_CONVERT, s);
        const cudaError_t le = launch_pdl(false, convert_bf16_f16_kernel, dim3(int(blocks)), dim3(256), 0, s, src,
                                          dst, n, err);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace moe

// selftest.cu — moe_wait_selftest: the bounded mbarrier wait of the pipelined
// kernels, run on a barrier that nothing completes. The wait must give up
// after its limit, raise MOE_DEVERR_TIMEOUT in the error word and let the
// kernel return, leaving the context usable. This checks the failure path on
// the GPU without faulting, trapping or hanging it.
#include "internal.h"

namespace moe {
namespace {

__global__ void __launch_bounds__(32) wait_selftest_kernel(uint32_t* err, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // expects one arrival that never comes
        abort_flag = 0;
        fence_mbar_init();
        mbar_wait_bounded(&bar, 0, &abort_flag, err, limit_ns);  // gives up after limit_ns
    }
}

}  // namespace
}  // namespace moe

extern "C" MOE_API int moe_wait_selftest(void* err_ws, uint64_t limit_ns, moe_stream_t stream) {
    using namespace moe;
    if (!err_ws) return MOE_ERR_INVALID_ARG;
    if (limit_ns == 0 || limit_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;  // at most 10 s
    wait_selftest_kernel<<<1, 32, 0, stream>>>(static_cast<uint32_t*>(err_ws), limit_ns);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

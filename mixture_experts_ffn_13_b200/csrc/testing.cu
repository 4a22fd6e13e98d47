// testing.cu -- moe_test_bounded_wait (include/moe_b200_testing.h): the library's bounded
// mbarrier wait, run on a barrier that nothing arrives at.
#include "../../include/moe_b200_testing.h"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

__global__ void bounded_wait_kernel(int *status, uint64_t timeout_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    // phase 0 of a fresh barrier with one expected arrival: never completes here
    mbar_wait(&bar, 0, &abort_flag, status, timeout_ns);
}

}  // namespace
}  // namespace moe

extern "C" int moe_test_bounded_wait(int32_t *status, int32_t timeout_us, moe_stream_t stream)
{
    if (!status || timeout_us < 1 || timeout_us > 1000000) return MOE_ERR_INVALID_ARG;
    moe::bounded_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(status, (uint64_t)timeout_us * 1000ull);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// moda_selftest.cu -- exercises the kernels' bounded-wait failure path.
//
// Every mbarrier wait in the forward and backward kernels gives up after a
// fixed time (or when another warp of the CTA has already given up), records
// kStatusTimeout in the device status word and lets the kernel return, so a
// lost arrival can never hang the GPU.  This launch makes that path run on
// purpose without any fault: one CTA of two warps waits on a freshly
// initialised mbarrier that nothing ever arrives on.  The first warp to time
// out raises the CTA's abort flag, the other leaves on the flag (or its own
// limit), and the kernel ends normally with the status word set.
#include <cuda_runtime.h>

#include "moda_internal.h"
#include "moda_ptx.cuh"

namespace moda {
namespace {

__global__ void __launch_bounds__(64) wait_timeout_selftest_kernel(unsigned int* status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        abort_flag = 0;
    }
    __syncthreads();
    if ((threadIdx.x & 31) == 0) {
        // phase 0 of a barrier expecting one arrival that never comes
        ptx::mbar_wait(&bar, 0, status, &abort_flag);
    }
    __syncthreads();
}

}  // namespace
}  // namespace moda

extern "C" moda_status moda_selftest_wait_timeout(moda_stream_t stream) {
    unsigned int* w = moda::device_status_word();
    if (!w) return moda::api_fail(MODA_ERR_CUDA, "no usable CUDA device");
    moda::wait_timeout_selftest_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(w);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MODA_OK : moda::api_fail(MODA_ERR_CUDA, cudaGetErrorString(e));
}

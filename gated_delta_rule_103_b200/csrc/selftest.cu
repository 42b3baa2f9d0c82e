// Self-test of the kernels' bounded wait: one CTA waits on an mbarrier that
// nothing arrives on, with the same wait routine the tensor-core kernels use
// but a short limit.  The wait runs out, records the timeout in the library's
// device error word and the kernel returns, leaving the context usable.  It
// lets a test check the failure path on a GPU without faulting or hanging it.
#include <cuda_runtime.h>

#include "chunk_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

__global__ void kda_wait_selftest_kernel(unsigned* err, unsigned long long limit_ns)
{
    __shared__ __align__(8) unsigned long long mbar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(ptx::smem_u32(&mbar), 1);
        ptx::fence_mbar_init();
        abort_flag = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // phase 0 never completes: no thread arrives and no copy is pending
        tc::wait_bar(ptx::smem_u32(&mbar), 0, &abort_flag, err, limit_ns);
    }
    __syncthreads();
}

}  // namespace

cudaError_t launch_wait_selftest(unsigned* err, unsigned long long limit_ns, cudaStream_t stream)
{
    kda_wait_selftest_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
    return cudaGetLastError();
}

}  // namespace kda

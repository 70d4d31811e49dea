// Diagnostic kernel: a bounded mbarrier wait that nothing completes.  It
// shows, on the device, the failure path every pipeline wait of this library
// takes -- give up after the wait limit, record a timeout in the per-device
// error word, return -- without faulting or hanging the GPU.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

__global__ void wait_timeout_kernel(uint32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);
    fence_mbar_init();
    abort_flag = 0;
  }
  __syncthreads();
  // no thread ever arrives on `bar`: the wait runs out after kWaitLimitNs
  if (threadIdx.x == 0) mbar_wait(smem_addr(&bar), 0, &abort_flag, err);
}

}  // namespace

dsa_status_t selftest_wait_timeout(uint32_t* err, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(err);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa

// moe_selftest_bounded_wait: a check of the failure path every kernel relies on.
//
// Each mbarrier wait in the library gives up after a wall-clock limit, reports
// MOE_ERR_TIMEOUT in the device status word and lets its kernel return, so that a
// lost arrival (a bug, or a peer that never comes) leaves the GPU usable instead of
// hanging it.  This entry point runs that wait, through the same mbar_wait_for the
// kernels use, on a barrier that nothing ever arrives at, with a limit the caller
// chooses: the wait must expire, set the status word and end the kernel.
#include "common.cuh"
#include "internal.h"

#include <nvtx3/nvToolsExt.h>

namespace moe {
namespace {

// One thread of one CTA: a barrier expecting one arrival that never comes.
__global__ void bounded_wait_kernel(uint64_t limit_ns, int* err, int* done) {
  __shared__ uint64_t bar;
  pdl_begin();
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  mbar_fence_init();
  const bool arrived = mbar_wait_for(b, 0, err, limit_ns);
  *done = arrived ? 2 : 1;   // 1: the wait expired and the kernel went on to its end
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_selftest_bounded_wait(uint64_t limit_ns, int32_t* done, void* stream) {
  nvtxRangePushA("moe_selftest_bounded_wait");
  moe_status_t st = MOE_OK;
  int* err = moe_status_word();
  if (limit_ns < 1000ull || limit_ns > kWaitLimitNs || done == nullptr) {
    st = MOE_ERR_INVALID_ARG;
  } else if (err == nullptr) {
    st = MOE_ERR_CUDA;
  } else {
    const cudaError_t e = launch_pdl(bounded_wait_kernel, dim3(1), dim3(1), 0,
                                     static_cast<cudaStream_t>(stream), 1, limit_ns, err,
                                     reinterpret_cast<int*>(done));
    st = (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? MOE_OK : MOE_ERR_CUDA;
  }
  nvtxRangePop();
  return st;
}

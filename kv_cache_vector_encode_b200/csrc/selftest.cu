// tq_selftest_wait: exercises the library's failure-detection path on the GPU without a fault.
//
// Every producer / consumer hand-off in the libtq kernels is an mbarrier wait bounded in time
// (sm100.cuh): a wait that runs out records a code in the library's device error word and the
// kernel returns, so a lost arrival shows up as TQ_ERR_DEVICE_TIMEOUT from tq_sync_check instead
// of a hung GPU. This self-test runs that exact wait on an mbarrier that nothing ever arrives on,
// with a short limit, so that a caller (or a test) can see the whole path work: the wait gives up,
// the error word is set, tq_sync_check reports and clears it, and the context stays usable.
#include <cuda_runtime.h>

#include <string>

#include "sm100.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

__global__ void selftest_wait_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);          // one expected arrival, which never comes
    abort_flag = 0u;
    fence_mbar_init();
  }
  __syncthreads();
  // the phase of parity 0 never completes: the bounded wait records kDevTimeoutSync and returns
  mbar_wait_warp(&bar, 0u, err, kDevTimeoutSync, &abort_flag, limit_ns);
}

}  // namespace
}  // namespace tq

extern "C" TQ_API tq_status tq_selftest_wait(uint64_t limit_ns, void* stream) {
  tq::clear_error();
  if (limit_ns < 1000u || limit_ns > tq::kWaitLimitNs)
    return tq::fail(TQ_ERR_INVALID_ARG, "tq_selftest_wait: limit_ns must lie in [1000, 1e9]");
  uint32_t* err = tq::device_error_word();
  if (!err) return tq::fail(TQ_ERR_CUDA, "tq_selftest_wait: no device error word");
  tq::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(err, limit_ns);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return tq::cuda_fail(e, "tq_selftest_wait: launch");
  return TQ_OK;
}

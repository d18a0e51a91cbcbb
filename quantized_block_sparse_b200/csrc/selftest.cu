// selftest.cu - a diagnostic launch that exercises the bounded-wait failure path.
//
// Every kernel of this library waits on mbarriers through mbar_wait, which gives up after a
// time limit, sets a bit in the caller's status word and lets the kernel return instead of
// hanging the GPU. The path only runs when something has gone wrong, so it needs a way to
// be tested on purpose without a fault: this kernel initialises one mbarrier that nothing
// will ever arrive on and waits on it through the same bounded wait with a short, caller-
// chosen limit. The wait runs out, the status word gets SAGESLA_ERR_TIMEOUT's bit, the kernel
// returns, and the context stays usable; sagesla_check_status then reports the timeout.
#include "../../include/sagesla.h"
#include "sagesla_internal.h"
#include "sm100_primitives.cuh"

namespace sgs {
namespace {

__global__ void __launch_bounds__(32) wait_selftest_kernel(int* status,
                                                           unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  // Phase 0 of `bar` never completes (its one expected arrival never comes): the wait ends
  // only through its time limit.
  mbar_wait_limit(smem_u32(&bar), 0, &abort_flag, status, limit_ns);
}

}  // namespace
}  // namespace sgs

extern "C" int sagesla_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                             unsigned int limit_us, void* stream) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 15u) || workspace_bytes < 256)
    return SAGESLA_ERR_INVALID_ARG;
  if (limit_us < 1 || limit_us > 1000000u) return SAGESLA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  {
    sgs::TraceScope ts_("wait_selftest_kernel", st);
    sgs::wait_selftest_kernel<<<1, 32, 0, st>>>(static_cast<int*>(workspace),
                                                1000ull * limit_us);
  }
  return cudaGetLastError() == cudaSuccess ? SAGESLA_OK : SAGESLA_ERR_CUDA;
}

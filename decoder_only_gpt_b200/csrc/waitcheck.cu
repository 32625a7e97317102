// Check of the failure path every pipeline kernel shares: a bounded mbarrier
// wait that expires records GPT_ETIMEOUT in the workspace status word and the
// kernel returns, leaving the context usable.  One thread waits on a barrier
// that nothing ever arrives at; nothing faults, traps or hangs.
#include <cuda_runtime.h>

#include "device_common.cuh"
#include "gpt_internal.h"
#include "tc_ptx.cuh"

namespace gpt {
namespace {

__global__ void wait_expiry_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !tc::mbar_wait_bounded(&bar, 0, nullptr, limit_ns))
    record_status(status, GPT_ETIMEOUT, K_WAITCHECK, 0);
}

}  // namespace

int launch_wait_expiry(int32_t* status, uint64_t limit_ns, void* stream) {
  wait_expiry_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(status, limit_ns);
  return last_launch_rc();
}

}  // namespace gpt

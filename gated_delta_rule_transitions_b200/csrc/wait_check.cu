// Bounded-wait check.  One kernel waits on a shared-memory mbarrier with the same
// bounded wait the tensor-core kernels use.  If the barrier is never completed, the
// wait gives up after the given limit, the timeout is recorded in this unit's device
// error word and the kernel returns; hla_device_status reports it as
// HLA_ERR_TIMEOUT.  It lets a caller see, on a real device, that an expired wait is
// reported and the context stays usable, with no fault and no hang.
#include "common.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"

namespace hla {

HLA_DEFINE_ERROR_WORD(wait_check)

namespace {

__global__ void wait_check_kernel(uint64_t limit_ns, int complete) {
  __shared__ uint64_t bar;
  __shared__ int abort_s;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    abort_s = 0;
    tc::mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (complete) tc::mbar_arrive(&bar);
    if (!tc::mbar_wait(&bar, 0, (volatile int*)&abort_s, limit_ns)) report_device_error(kErrMbarTimeout);
  }
}

}  // namespace

cudaError_t launch_wait_check(uint64_t limit_ns, bool complete, cudaStream_t s) {
  wait_check_kernel<<<1, 32, 0, s>>>(limit_ns, complete ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace hla

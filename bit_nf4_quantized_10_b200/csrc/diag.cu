// Self-test of the bounded waits that every pipelined kernel relies on: one
// CTA waits on an mbarrier that nothing arrives on, through the same wait the
// kernels use.  The wait gives up after its poll limit, records a timeout in
// the status word and the kernel returns, so the context stays usable.
#include "common.cuh"
#include "sm100.cuh"
#include "trace.cuh"

namespace ql {
using namespace sm100;

QL_DEFINE_STATUS_ACCESSOR(status_word_diag)

__global__ void wait_timeout_kernel(uint32_t polls) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, polls);   // no arrival: runs out
  __syncthreads();
}

ql_status launch_wait_timeout(uint32_t polls, cudaStream_t st) {
  QL_CUDA_TRY(launch(wait_timeout_kernel, dim3(1), dim3(32), 0, st, 1, 1, polls));
  return QL_OK;
}

}  // namespace ql

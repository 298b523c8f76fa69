// Failure detection without a GPU fault: a kernel whose threads wait, with the
// library's bounded mbarrier wait, on a barrier that nothing ever completes.
// CTA 0 gives up after `limit` cycles and records REST_ERR_TIMEOUT in the
// status word; every other CTA waits with the library's own (about one
// second) bound and gives up as soon as it sees that word, as the CTAs of any
// library kernel do when one of them has failed. The kernel then returns and
// the context stays usable.
#include "kernels.h"
#include "sm100.h"
#include "sm100_common.cuh"

namespace rest {
namespace {

using namespace sm100;

__global__ void wait_timeout_kernel(int32_t* err, long long limit) {
  pdl_wait();
  pdl_release();
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  mbar_wait_for(&bar, 0, err, &abort_flag, blockIdx.x == 0 ? limit : kWaitCycles);
}

}  // namespace

cudaError_t launch_wait_timeout(int n_ctas, long long limit_cycles, int32_t* err, cudaStream_t s) {
  return launch_k(wait_timeout_kernel, n_ctas, 128, 0, s, err, limit_cycles);
}

}  // namespace rest

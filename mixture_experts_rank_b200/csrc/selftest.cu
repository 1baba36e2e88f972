// Self-test of the kernels' failure path: one bounded mbarrier wait that nothing completes.
// The wait gives up after its time limit, records MORE_DEVERR_WAIT_TIMEOUT in the device error
// word and returns, so the context stays usable.  Every persistent kernel of the library waits
// through the same bounded_wait.
#include "mbar_wait.cuh"
#include "more_internal.cuh"

namespace more {
namespace {

__global__ void wait_timeout_probe_kernel(unsigned int* status, int32_t* out_result) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  sm100::mbar_init(&bar, 1);
  sm100::fence_mbar_init();
  abort_flag = 0;
  // nothing arrives on bar: the wait runs out after sm100::kWaitLimitNs
  const bool completed = sm100::bounded_wait(&bar, 0, &abort_flag, status);
  *out_result = completed ? 1 : 2;
}

}  // namespace

cudaError_t launch_wait_timeout_probe(unsigned int* status, int32_t* out_result, cudaStream_t stream) {
  wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(status, out_result);
  return cudaGetLastError();
}

}  // namespace more

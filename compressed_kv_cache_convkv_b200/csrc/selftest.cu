// Self-test of the bounded barrier wait every kernel of the library uses.
//
// One CTA waits on an mbarrier that nothing ever arrives on.  The wait must give
// up after its clock budget, raise the CTA's abort flag and let the kernel
// record CONVKV_ERR_DEVICE_TIMEOUT in a status word, so a stalled pipeline ends
// as an error the host can read instead of a hung GPU.  No trap, no fault.
#include "../../include/convkv.h"
#include "convkv_internal.h"
#include "sm100.cuh"

namespace ckv {
namespace {

__global__ void wait_timeout_selftest_kernel(int* status, long long budget) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    dev::mbar_init(&bar, 1);
    abort_flag = 0;
    dev::fence_mbar_init();
  }
  __syncthreads();
  const bool ok = dev::mbar_wait(&bar, 0, &abort_flag, budget);  // never completes
  __syncthreads();
  if (threadIdx.x == 0 && (!ok || abort_flag)) atomicExch(status, kStatusTimeout);
}

}  // namespace
}  // namespace ckv

extern "C" int convkv_selftest_wait_timeout(int* dev_status, long long budget_clocks, void* stream) {
  if (!dev_status || budget_clocks < 1000 || budget_clocks > ckv::dev::kWaitBudgetClocks) return CONVKV_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ckv::wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(dev_status, budget_clocks);
  if (cudaGetLastError() != cudaSuccess) return CONVKV_ERR_CUDA;
  int st = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return CONVKV_ERR_CUDA;
  if (cudaMemcpy(&st, dev_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return CONVKV_ERR_CUDA;
  return st == ckv::kStatusTimeout ? CONVKV_ERR_DEVICE_TIMEOUT : CONVKV_OK;
}

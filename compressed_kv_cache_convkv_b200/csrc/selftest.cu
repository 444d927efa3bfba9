// Self-test of the bounded barrier wait every kernel of the library uses.
//
// One CTA waits on an mbarrier that nothing ever arrives on.  The wait must give
// up after its clock budget, raise the CTA's abort flag and let the kernel
// record CONVKV_ERR_DEVICE_TIMEOUT in a status word, so a stalled pipeline ends
// as an error the host can read instead of a hung GPU.  No trap, no fault.
#include <algorithm>

#include "../../include/convkv.h"
#include "convkv_internal.h"
#include "quant_div.cuh"
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

// div_rn (the quantisers' shared-divisor quotient) against CUDA's IEEE division,
// bit for bit, over caller-supplied pairs.
__global__ void div_rn_selftest_kernel(const float* x, const float* s, int64_t n, unsigned int* mismatches) {
  unsigned int bad = 0;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float a = x[i], b = s[i];
    const float got = div_rn(a, make_divisor(b));
    const float want = __fdiv_rn(a, b);
    const bool same = __float_as_uint(got) == __float_as_uint(want) || (got != got && want != want);
    bad += same ? 0u : 1u;
  }
  for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
  if ((threadIdx.x & 31) == 0 && bad) atomicAdd(mismatches, bad);
}

}  // namespace
}  // namespace ckv

extern "C" int convkv_selftest_div_rn(const float* dev_x, const float* dev_s, int64_t n, unsigned int* dev_mismatches,
                                      void* stream) {
  if (!dev_x || !dev_s || !dev_mismatches || n < 0) return CONVKV_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n > 0) {
    const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 16);
    ckv::div_rn_selftest_kernel<<<static_cast<int>(blocks), 256, 0, st>>>(dev_x, dev_s, n, dev_mismatches);
    if (cudaGetLastError() != cudaSuccess) return CONVKV_ERR_CUDA;
  }
  if (cudaStreamSynchronize(st) != cudaSuccess) return CONVKV_ERR_CUDA;
  return CONVKV_OK;
}

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

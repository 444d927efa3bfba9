// Seeded synthetic inputs, device side.
//
// Same generator and transform as gen_host.c (Philox4x32-10 from its published
// definition, Irwin-Hall(12) from twelve 10-bit uniforms, one IEEE
// round-to-nearest fp32 multiply, bf16 round-to-nearest-even), so that a value
// produced here is bit-identical to the host value at the same
// (seed, tensor, state, frame, element).  Holds no arithmetic of the method.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;

__device__ __forceinline__ uint16_t value_bf16(uint32_t seed, uint32_t tensor, uint32_t state,
                                               uint32_t frame, uint32_t elem, float scale) {
  uint32_t c0 = elem, c1 = frame, c2 = state, c3 = tensor;
  uint32_t k0 = seed, k1 = 0u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) { k0 += kW0; k1 += kW1; }
    uint32_t lo0 = kM0 * c0, hi0 = __umulhi(kM0, c0);
    uint32_t lo1 = kM1 * c2, hi1 = __umulhi(kM1, c2);
    uint32_t n0 = hi1 ^ c1 ^ k0;
    uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
  }
  uint32_t w[4] = {c0, c1, c2, c3};
  int32_t sum = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    sum += (int32_t)(w[i] & 1023u) + (int32_t)((w[i] >> 10) & 1023u) + (int32_t)((w[i] >> 20) & 1023u);
  float x = __fmul_rn((float)(sum - 6138), 1.0f / 1024.0f);
  float xs = __fmul_rn(x, scale);
  uint32_t u = __float_as_uint(xs);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

__global__ void fill_kernel(uint16_t* out, uint32_t seed, uint32_t tensor, uint32_t state,
                            uint32_t frame0, uint64_t frame_elems, uint64_t total, float scale) {
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    uint32_t f = (uint32_t)(i / frame_elems);
    uint32_t e = (uint32_t)(i - (uint64_t)f * frame_elems);
    out[i] = value_bf16(seed, tensor, state, frame0 + f, e, scale);
  }
}

}  // namespace

// Fills out[f * frame_elems + e] for f < nframes, e < frame_elems on `stream`.
// Returns the cudaError_t of the launch (0 on success).
extern "C" int si_fill_bf16_device(void* out, uint32_t seed, uint32_t tensor, uint32_t state,
                                   uint32_t frame0, uint32_t nframes, uint64_t frame_elems,
                                   float scale, void* stream) {
  uint64_t total = (uint64_t)nframes * frame_elems;
  if (total == 0) return 0;
  if (out == nullptr) return (int)cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  uint64_t want = (total + 255) / 256;
  uint64_t cap = (uint64_t)sms * 16;
  unsigned grid = (unsigned)(want < cap ? want : cap);
  fill_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>((uint16_t*)out, seed, tensor, state, frame0,
                                                      frame_elems, total, scale);
  return (int)cudaGetLastError();
}

// e4m3 quantisation of bf16 frames that allocates no device memory.
//
// Some callers cannot allocate device memory while they run: a serving engine
// that hands out every device byte from its own fixed pool, or a thread on a
// latency-critical path where cudaMalloc would synchronise the device and stall
// its other streams.  This entry point needs no handle and no arena.  It does
// the same quantisation as the fp8 append (per frame and head: scale =
// amax / 448, code = e4m3(x / scale), IEEE fp32 divide, round-to-nearest-even,
// saturating), and its only scratch -- one amax per (frame, head) -- lives in
// the fixed array below, which every GPU that loads this library keeps until
// the process exits.
#include <mutex>

#include "../../include/convkv.h"
#include "convkv_internal.h"

namespace {

constexpr int kMaxFrameHeads = CONVKV_NOALLOC_MAX_FRAME_HEADS;

// The scratch.  Host code must not pass this name to a kernel: on the host it is
// only a stand-in for the symbol; the device address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned int g_noalloc_amax[kMaxFrameHeads];

constexpr int kMaxDevices = 128;
std::mutex g_mu;
unsigned int* g_amax_addr[kMaxDevices] = {};

int grid_cap(int64_t items, int threads) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t want = (items + threads - 1) / threads;
  int64_t cap = static_cast<int64_t>(sms) * 8;
  if (want < 1) want = 1;
  return static_cast<int>(want < cap ? want : cap);
}

// amax over each frame's [tokens, head_dim] values per head; grid = (row splits, frames)
__global__ void noalloc_amax_kernel(const uint4* __restrict__ x, unsigned int* __restrict__ amax, int tokens,
                                    int heads, int head_dim, int rows_per_block) {
  extern __shared__ unsigned int sh[];
  const int f = blockIdx.y;
  for (int h = threadIdx.x; h < heads; h += blockDim.x) sh[h] = 0;
  __syncthreads();
  const int vec_per_row = heads * head_dim / 8;
  const int64_t frame_vecs = static_cast<int64_t>(tokens) * vec_per_row;
  const int r0 = blockIdx.x * rows_per_block;
  const int r1 = min(tokens, r0 + rows_per_block);
  const uint4* src = x + f * frame_vecs;
  for (int64_t i = static_cast<int64_t>(r0) * vec_per_row + threadIdx.x; i < static_cast<int64_t>(r1) * vec_per_row;
       i += blockDim.x) {
    const uint4 v = __ldg(src + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t m = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      m = max(m, (w[q] & 0x7FFFu) << 16);
      m = max(m, w[q] & 0x7FFF0000u);
    }
    atomicMax(&sh[(i % vec_per_row) * 8 / head_dim], m);
  }
  __syncthreads();
  for (int h = threadIdx.x; h < heads; h += blockDim.x)
    if (sh[h]) atomicMax(&amax[f * heads + h], sh[h]);
}

__global__ void noalloc_quant_kernel(const uint4* __restrict__ x, const unsigned int* __restrict__ amax,
                                     uint2* __restrict__ codes, float* __restrict__ scales, int64_t total,
                                     int tokens, int heads, int head_dim) {
  const int vec_per_row = heads * head_dim / 8;
  const int64_t frame_vecs = static_cast<int64_t>(tokens) * vec_per_row;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int f = static_cast<int>(i / frame_vecs);
    const int64_t e = i - f * frame_vecs;
    const int h = static_cast<int>((e % vec_per_row) * 8 / head_dim);
    const float a = __uint_as_float(amax[f * heads + h]);
    const float scale = a > 0.0f ? __fdiv_rn(a, 448.0f) : 1.0f;
    const uint4 v = __ldg(x + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint16_t lo, hi;
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
          : "=h"(lo)
          : "f"(__fdiv_rn(__uint_as_float(w[2 * q] & 0xFFFF0000u), scale)),
            "f"(__fdiv_rn(__uint_as_float(w[2 * q] << 16), scale)));
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
          : "=h"(hi)
          : "f"(__fdiv_rn(__uint_as_float(w[2 * q + 1] & 0xFFFF0000u), scale)),
            "f"(__fdiv_rn(__uint_as_float(w[2 * q + 1] << 16), scale)));
      o[q] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    }
    codes[i] = make_uint2(o[0], o[1]);
    if (e < vec_per_row && (e * 8) % head_dim == 0) scales[f * heads + h] = scale;
  }
}

}  // namespace

extern "C" int convkv_quantize_e4m3_noalloc(const void* x, void* codes, float* scales, int frames, int tokens,
                                            int heads, int head_dim, void* stream) {
  if (!x || !codes || !scales || frames < 1 || tokens < 1 || heads < 1 || head_dim < 8 || head_dim % 8)
    return CONVKV_ERR_INVALID_ARG;
  // the kernels read x in 16-byte vectors, write codes in 8-byte vectors and scales as fp32
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(codes) & 7u) ||
      (reinterpret_cast<uintptr_t>(scales) & 3u))
    return CONVKV_ERR_INVALID_ARG;
  if (static_cast<int64_t>(frames) * heads > kMaxFrameHeads) return CONVKV_ERR_SCRATCH_LIMIT;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return CONVKV_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return CONVKV_ERR_UNSUPPORTED;
  unsigned int* amax = nullptr;
  {
    // first call on this device: resolve the array's device address (with this device
    // current); the address stays valid for the life of the primary context, so a
    // cudaDeviceReset after this call is not supported
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_amax_addr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_amax);
      if (e != cudaSuccess || !p) return CONVKV_ERR_CUDA;
      g_amax_addr[dev] = static_cast<unsigned int*>(p);
    }
    amax = g_amax_addr[dev];
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the array keeps the previous call's values: clear the part this call reduces into
  e = cudaMemsetAsync(amax, 0, sizeof(unsigned int) * frames * heads, s);
  if (e != cudaSuccess) return CONVKV_ERR_CUDA;
  const int rows_per_block = 64;
  dim3 g1((tokens + rows_per_block - 1) / rows_per_block, frames);
  noalloc_amax_kernel<<<g1, 256, heads * sizeof(unsigned int), s>>>(static_cast<const uint4*>(x), amax, tokens,
                                                                    heads, head_dim, rows_per_block);
  if (cudaGetLastError() != cudaSuccess) return CONVKV_ERR_CUDA;
  const int64_t total = static_cast<int64_t>(frames) * tokens * heads * head_dim / 8;
  noalloc_quant_kernel<<<grid_cap(total, 256), 256, 0, s>>>(static_cast<const uint4*>(x), amax,
                                                            static_cast<uint2*>(codes), scales, total, tokens, heads,
                                                            head_dim);
  if (cudaGetLastError() != cudaSuccess) return CONVKV_ERR_CUDA;
  return CONVKV_OK;
}

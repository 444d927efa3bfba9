// Streaming kernels: append of a block into the ring (bf16), permutation of the
// conv weights into the compression kernel's layout, and the mean-of-5
// compression variant.  All HBM-bound: 16-byte vector accesses, grids sized as
// a multiple of the SM count.
#include "convkv_internal.h"

namespace ckv {
namespace {

int grid_for(int64_t work_items, int threads) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t want = (work_items + threads - 1) / threads;
  int64_t cap = static_cast<int64_t>(sms) * 8;
  if (want < 1) want = 1;
  return static_cast<int>(want < cap ? want : cap);
}

// Append (SoulX-LiveAct blog, "ConvKV Memory": append-only KV -- only the new
// tokens' K/V are written, cached entries are never recomputed).
// k, v: [S][b*T][H][D] bf16 -> ring slot (slot0 + f) % R of each state.
__global__ void append_bf16_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                   uint4* __restrict__ ringK, uint4* __restrict__ ringV, AppendParams p) {
  const int64_t fv = p.frame_elems / 8;  // 16-byte vectors per frame
  const int64_t total = static_cast<int64_t>(p.S) * p.b * fv;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int64_t sf = i / fv;               // state * b + f
    const int64_t e = i - sf * fv;
    const int s = static_cast<int>(sf / p.b);
    const int f = static_cast<int>(sf - static_cast<int64_t>(s) * p.b);
    int slot = p.slot0 + f;
    if (slot >= p.R) slot -= p.R;
    const int64_t dst = (static_cast<int64_t>(s) * p.R + slot) * fv + e;
    const uint4 kv = __ldcs(k + i);
    const uint4 vv = __ldcs(v + i);
    ringK[dst] = kv;
    ringV[dst] = vv;
  }
}

// [S][2][H][D_out][D_in][5] -> [S][2][H][5][D_out][D_in]
__global__ void permute_weights_kernel(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                       int64_t n, int D) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    // i indexes the destination
    const int in_ = static_cast<int>(i % D);
    const int64_t r1 = i / D;
    const int o = static_cast<int>(r1 % D);
    const int64_t r2 = r1 / D;
    const int j = static_cast<int>(r2 % kEvict);
    const int64_t skh = r2 / kEvict;  // (s * 2 + kv) * H + h
    const int64_t src_idx = ((skh * D + o) * D + in_) * kEvict + j;
    dst[i] = src[src_idx];
  }
}

// Mean of the 5 evicted frames (the model card's --mean_memory option):
// out = bf16(sum_j x_j / 5) with the sum and divide in fp32.
__global__ void mean_bf16_kernel(const uint4* __restrict__ ringK, const uint4* __restrict__ ringV,
                                 uint4* __restrict__ memK, uint4* __restrict__ memV, ConvParams p,
                                 int64_t frame_vecs) {
  const int64_t per_group = static_cast<int64_t>(p.S) * frame_vecs * 2;
  const int64_t total = per_group * p.ngroups;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int g = static_cast<int>(i / per_group);
    int64_t r = i - g * per_group;
    const int kv = static_cast<int>(r / (static_cast<int64_t>(p.S) * frame_vecs));
    r -= static_cast<int64_t>(kv) * p.S * frame_vecs;
    const int s = static_cast<int>(r / frame_vecs);
    const int64_t e = r - static_cast<int64_t>(s) * frame_vecs;
    const uint4* src = kv ? ringV : ringK;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < kEvict; ++j) {
      const uint4 x = src[(static_cast<int64_t>(s) * p.R + p.grp[g].ring_slot[j]) * frame_vecs + e];
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[2 * q] += __uint_as_float(w[q] << 16);
        acc[2 * q + 1] += __uint_as_float(w[q] & 0xFFFF0000u);
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      __nv_bfloat162 h2 = __floats2bfloat162_rn(__fdiv_rn(acc[2 * q], 5.0f), __fdiv_rn(acc[2 * q + 1], 5.0f));
      o[q] = *reinterpret_cast<uint32_t*>(&h2);
    }
    uint4* dst = kv ? reinterpret_cast<uint4*>(p.memV) : reinterpret_cast<uint4*>(p.memK);
    dst[(static_cast<int64_t>(s) * p.C + p.grp[g].mem_pos) * frame_vecs + e] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

int launch_append_bf16(const AppendParams& p, const void* k, const void* v, void* ringK, void* ringV,
                       cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(p.S) * p.b * (p.frame_elems / 8);
  append_bf16_kernel<<<grid_for(total, 256), 256, 0, s>>>(static_cast<const uint4*>(k), static_cast<const uint4*>(v),
                                                          static_cast<uint4*>(ringK), static_cast<uint4*>(ringV), p);
  return static_cast<int>(cudaGetLastError());
}

int launch_permute_weights(const void* src, void* dst, int S, int H, int D, cudaStream_t s) {
  const int64_t n = static_cast<int64_t>(S) * 2 * H * kEvict * D * D;
  permute_weights_kernel<<<grid_for(n, 256), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(src),
                                                          static_cast<__nv_bfloat16*>(dst), n, D);
  return static_cast<int>(cudaGetLastError());
}

int launch_mean_bf16(int D, const ConvParams& p, const void* ringK, const void* ringV, cudaStream_t s) {
  const int64_t frame_vecs = static_cast<int64_t>(p.T) * p.H * D / 8;
  const int64_t total = frame_vecs * p.S * 2 * p.ngroups;
  mean_bf16_kernel<<<grid_for(total, 256), 256, 0, s>>>(static_cast<const uint4*>(ringK),
                                                        static_cast<const uint4*>(ringV), static_cast<uint4*>(p.memK),
                                                        static_cast<uint4*>(p.memV), p, frame_vecs);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace ckv

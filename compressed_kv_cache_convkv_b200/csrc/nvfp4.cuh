// NVFP4 storage of the K/V cache: e2m1 codes (two per byte, the even channel in
// the low nibble), one e4m3 scale per 16 consecutive channels of a token, one
// fp32 scale g per (state, K|V, frame or slot, head).
//
//   g   = amax / (448 * 6) over the frame's [T, D] values of the head (1 if 0)
//   s_b = e4m3(a_b / (g * 6)), a_b = max |x| over block b
//   e_b = s_b * g,  code = e2m1(x / e_b)   (0 where e_b == 0)
//   value on use = bf16(code * e_b)
//
// every product and quotient rounded to nearest in fp32; e4m3 and e2m1 round to
// nearest even and saturate (model card, open-source plan: FP4 for B-series
// GPUs, read as the NVFP4 format; stored and dequantised to BF16 on use like
// the FP8 cache).
#pragma once
#include <cuda_fp16.h>

#include "convkv_internal.h"
#include "quant_div.cuh"
#include "sm100.cuh"

namespace ckv {
namespace fp4 {

constexpr int kBlock = 16;
constexpr float kRange = 448.0f * 6.0f;

// one e4m3 code (low byte of `code`) -> fp32 (exact)
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h2;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h2) : "r"(code & 0xFFu));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}
// fp32 -> e4m3 code (round to nearest even, saturating)
__device__ __forceinline__ uint32_t f32_to_e4m3(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;
}
// byte of two e2m1 codes -> (even channel, odd channel) as fp32 (exact)
__device__ __forceinline__ void e2m1x2_to_f32(uint32_t byte, float& lo, float& hi) {
  uint32_t h2;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h2) : "r"(byte & 0xFFu));
  lo = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
  hi = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
}
// (even, odd) fp32 -> byte of two e2m1 codes (round to nearest even, saturating)
__device__ __forceinline__ uint32_t f32x2_to_e2m1(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float tensor_scale(float amax) { return amax > 0.0f ? __fdiv_rn(amax, kRange) : 1.0f; }

// Block scale code of a block with max |x| = a_b under tensor scale g, and the
// effective scale e_b = s_b * g it stands for.
// g6 is the shared divisor g * 6 (rounded), built once per tensor scale.
__device__ __forceinline__ uint32_t block_scale(float a_b, float g, const SharedDivisor& g6, float& e_b) {
  const uint32_t s = f32_to_e4m3(div_rn(a_b, g6));
  e_b = __fmul_rn(e4m3_to_f32(s), g);
  return s;
}
__device__ __forceinline__ SharedDivisor block_divisor(float g) { return make_divisor(__fmul_rn(g, 6.0f)); }

// 16 values of one block -> 8 code bytes (as two 32-bit words each holding 4 bytes)
__device__ __forceinline__ uint2 encode_block(const float (&x)[kBlock], float e_b) {
  uint32_t w[2] = {0, 0};
  if (e_b > 0.0f) {
    const SharedDivisor d = make_divisor(e_b);
#pragma unroll
    for (int j = 0; j < kBlock / 2; ++j) {
      const uint32_t b = f32x2_to_e2m1(div_rn(x[2 * j], d), div_rn(x[2 * j + 1], d));
      w[j >> 2] |= b << (8 * (j & 3));
    }
  }
  return make_uint2(w[0], w[1]);
}

// 4 code bytes (8 channels) -> 4 bf16x2 words of code * e_b
__device__ __forceinline__ void decode8(uint32_t word, float e_b, uint32_t (&o)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float a, b;
    e2m1x2_to_f32(word >> (8 * q), a, b);
    o[q] = dev::pack_bf16x2(a * e_b, b * e_b);
  }
}

}  // namespace fp4
}  // namespace ckv

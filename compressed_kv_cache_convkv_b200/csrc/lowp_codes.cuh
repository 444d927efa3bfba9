// Widening of e4m3 and e2m1 codes without conversion instructions (which share the
// narrow pipe with the softmax's exponentials): the code's bits are moved into an
// fp32 bit pattern whose value is the code times a fixed power of two, and the scale
// that multiplies it carries the inverse power, so each product -- and its rounding
// to nearest -- is exactly code * scale.
#pragma once
#include "sm100.cuh"

namespace ckv {
namespace dev {

// Four e4m3 codes (one per byte of w) -> their values times 2^-120 as fp32: the code's
// 4-bit exponent field lands in the low bits of the fp32 exponent field and its 3
// mantissa bits on top of the fp32 mantissa, so a normal code 2^(e-7)(1+m/8) reads as
// 2^(e-127)(1+m/8) and a subnormal code m 2^-9 as the fp32 denormal m 2^-129; zero
// stays zero.  lo = (byte 0, byte 1), hi = (byte 2, byte 3).
__device__ __forceinline__ void e4m3x4_scaled(uint32_t w, uint64_t& lo, uint64_t& hi) {
  const uint32_t a0 = ((w << 20) & 0x07F00000u) | ((w << 24) & 0x80000000u);
  const uint32_t a1 = ((w << 12) & 0x07F00000u) | ((w << 16) & 0x80000000u);
  const uint32_t a2 = ((w << 4) & 0x07F00000u) | ((w << 8) & 0x80000000u);
  const uint32_t a3 = ((w >> 4) & 0x07F00000u) | (w & 0x80000000u);
  lo = f2_make(__uint_as_float(a0), __uint_as_float(a1));
  hi = f2_make(__uint_as_float(a2), __uint_as_float(a3));
}

// The two halves of an f16x2 word -> their values times 2^-112 as fp32 (exact for
// normal halves and zero; every e2m1 value is one).
__device__ __forceinline__ uint64_t f16x2_scaled(uint32_t h2) {
  const uint32_t lo = ((h2 << 13) & 0x0FFFE000u) | ((h2 << 16) & 0x80000000u);
  const uint32_t hi = ((h2 >> 3) & 0x0FFFE000u) | (h2 & 0x80000000u);
  return f2_make(__uint_as_float(lo), __uint_as_float(hi));
}

// Scales below which the fold stays exact: sc * 2^120 (e4m3) and e_b * 2^112 (NVFP4)
// must stay finite in fp32.  Larger scales multiply by the power of two first (exact)
// and by the scale second.
constexpr float kE4m3FoldLimit = 128.0f;
constexpr float kFp4FoldLimit = 32768.0f;
constexpr float kTwo120 = 1.329227995784916e36f;  // 2^120
constexpr float kTwo112 = 5.192296858534828e33f;  // 2^112

// Eight e4m3 codes (w0: channels 0-3, w1: channels 4-7) -> four bf16x2 words of
// bf16(fp32(code * sc)): the widened values times m1, then (unless fold) times m2.
// fold: m1 = sc * 2^120 (sc < kE4m3FoldLimit); else m1 = 2^120 (exact) and m2 = sc.
__device__ __forceinline__ void e4m3x8_to_bf16(uint32_t w0, uint32_t w1, uint64_t m1, bool fold, uint64_t m2,
                                               uint32_t (&o)[4]) {
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    uint64_t lo, hi;
    e4m3x4_scaled(k ? w1 : w0, lo, hi);
    lo = f2_mul(lo, m1);
    hi = f2_mul(hi, m1);
    if (!fold) {
      lo = f2_mul(lo, m2);
      hi = f2_mul(hi, m2);
    }
    float a, b;
    f2_split(lo, a, b);
    o[2 * k] = pack_bf16x2(a, b);
    f2_split(hi, a, b);
    o[2 * k + 1] = pack_bf16x2(a, b);
  }
}

// Eight e2m1 codes (4 bytes, even channel in the low nibble) -> four bf16x2 words of
// bf16(fp32(code * e_b)): fold: m1 = e_b * 2^112 (e_b < kFp4FoldLimit); else m1 =
// 2^112 (exact) and m2 = e_b.
__device__ __forceinline__ void e2m1x8_to_bf16(uint32_t word, uint64_t m1, bool fold, uint64_t m2,
                                               uint32_t (&o)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t h2;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(h2)
        : "r"((word >> (8 * q)) & 0xFFu));
    uint64_t v = f2_mul(f16x2_scaled(h2), m1);
    if (!fold) v = f2_mul(v, m2);
    float a, b;
    f2_split(v, a, b);
    o[q] = pack_bf16x2(a, b);
  }
}

}  // namespace dev
}  // namespace ckv

// Widening of e4m3 and e2m1 codes without conversion instructions (which share the
// narrow pipe with the softmax's exponentials): the code's bits are moved into an
// fp32 bit pattern whose value is the code times a fixed power of two, and the scale
// that multiplies it carries the inverse power, so each product -- and its rounding
// to nearest -- is exactly code * scale.
#pragma once
#include "sm100.cuh"

namespace ckv {
namespace dev {

// Four e4m3 codes (one per byte of w) -> their values times 2^-120 as fp32 bit
// patterns: the code's 4-bit exponent field lands in the low bits of the fp32
// exponent field and its 3 mantissa bits on top of the fp32 mantissa, so a normal
// code 2^(e-7)(1+m/8) reads as 2^(e-127)(1+m/8) and a subnormal code m 2^-9 as the
// fp32 denormal m 2^-129; zero stays zero.
__device__ __forceinline__ void e4m3x4_scaled(uint32_t w, float (&a)[4]) {
  a[0] = __uint_as_float(((w << 20) & 0x07F00000u) | ((w << 24) & 0x80000000u));
  a[1] = __uint_as_float(((w << 12) & 0x07F00000u) | ((w << 16) & 0x80000000u));
  a[2] = __uint_as_float(((w << 4) & 0x07F00000u) | ((w << 8) & 0x80000000u));
  a[3] = __uint_as_float(((w >> 4) & 0x07F00000u) | (w & 0x80000000u));
}

// The two halves of an f16x2 word -> their values times 2^-112 as fp32 (exact for
// normal halves and zero; every e2m1 value is one).
__device__ __forceinline__ void f16x2_scaled(uint32_t h2, float& lo, float& hi) {
  lo = __uint_as_float(((h2 << 13) & 0x0FFFE000u) | ((h2 << 16) & 0x80000000u));
  hi = __uint_as_float(((h2 >> 3) & 0x0FFFE000u) | (h2 & 0x80000000u));
}

// Scales below which the fold stays exact: sc * 2^120 (e4m3) and e_b * 2^112 (NVFP4)
// must stay finite in fp32.  Larger scales multiply by the power of two first (exact)
// and by the scale second.
constexpr float kE4m3FoldLimit = 128.0f;
constexpr float kFp4FoldLimit = 32768.0f;
constexpr float kTwo120 = 1.329227995784916e36f;  // 2^120
constexpr float kTwo112 = 5.192296858534828e33f;  // 2^112

// Eight e4m3 codes (w0: channels 0-3, w1: channels 4-7) -> four bf16x2 words of
// bf16(fp32(code * sc)).  FOLD: m = sc * 2^120 (sc < kE4m3FoldLimit), one product per
// value; otherwise m = sc and the power of two is multiplied out first (exact).
template <bool FOLD>
__device__ __forceinline__ void e4m3x8_to_bf16(uint32_t w0, uint32_t w1, float m, uint32_t (&o)[4]) {
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    float a[4];
    e4m3x4_scaled(k ? w1 : w0, a);
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = FOLD ? a[i] * m : (a[i] * kTwo120) * m;
    o[2 * k] = pack_bf16x2(a[0], a[1]);
    o[2 * k + 1] = pack_bf16x2(a[2], a[3]);
  }
}

// Eight e2m1 codes (4 bytes, even channel in the low nibble) -> four bf16x2 words of
// bf16(fp32(code * e_b)).  FOLD: m = e_b * 2^112 (e_b < kFp4FoldLimit); otherwise
// m = e_b and the power of two is multiplied out first (exact).
template <bool FOLD>
__device__ __forceinline__ void e2m1x8_to_bf16(uint32_t word, float m, uint32_t (&o)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t h2;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(h2)
        : "r"((word >> (8 * q)) & 0xFFu));
    float a, b;
    f16x2_scaled(h2, a, b);
    a = FOLD ? a * m : (a * kTwo112) * m;
    b = FOLD ? b * m : (b * kTwo112) * m;
    o[q] = pack_bf16x2(a, b);
  }
}

}  // namespace dev
}  // namespace ckv

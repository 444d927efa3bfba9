// 3D RoPE on the fly: the rotation of adjacent channel pairs (2i, 2i+1) of each
// axis segment [t | h | w] of a head by tabulated angles, shared by the attention
// kernel (keys and queries) and the append (keys stored pre-rotated).
// (SoulX-LiveAct: RoPE Reset in the press article and the aiboss88.com summary;
// the split of D over the t, h, w axes and the frequencies are readings of the
// pages: h = w = 2 floor(D/6) channels, t the rest, frequency theta^(-2i/d_axis).)
#pragma once
#include "convkv_internal.h"
#include "sm100.cuh"

namespace ckv {

template <int D>
struct RopeCfg {
  static constexpr int PT = rope_pairs_t(D);  // rotation pairs on the time axis
  static constexpr int PH = rope_pairs_h(D);  // ... on the row axis
  static constexpr int PW = rope_pairs_h(D);  // ... on the column axis
  // 16-byte table units per position of each axis
  static constexpr int UT = rope_units(0, PT), UH = rope_units(PT, PH), UW = rope_units(PT + PH, PW);
  // axis (0 t, 1 h, 2 w) of global pair p, and the unit that holds it
  static constexpr int axis_of(int p) { return p < PT ? 0 : (p < PT + PH ? 1 : 2); }
  static constexpr int axis_start(int a) { return a == 0 ? 0 : (a == 1 ? PT : PT + PH); }
  static constexpr int unit_of(int p) { return p / 2 - axis_start(axis_of(p)) / 2; }
};

namespace dev {

// Row pointers into the three RoPE tables for one token position (t, y, x).
struct RopeRow {
  const float4* t;
  const float4* h;
  const float4* w;
  __device__ __forceinline__ float4 unit(int axis, int u) const {
    return __ldg((axis == 0 ? t : (axis == 1 ? h : w)) + u);
  }
};

__device__ __forceinline__ uint32_t rot_pair(uint32_t word, float c, float s, float scale, bool do_scale) {
  const float a = bf16lo_to_f32(word), b = bf16hi_to_f32(word);
  float ra = a * c - b * s, rb = a * s + b * c;
  if (do_scale) {
    ra *= scale;
    rb *= scale;
  }
  return pack_bf16x2(ra, rb);
}

// Rotate the 8 channels (4 adjacent pairs) of chunk c, held as bf16x2 words, in
// place.  Two pairs of the same axis go through packed fp32x2 arithmetic with one
// 16-byte table load; a pair-pair split by an axis boundary is rotated pair by pair.
template <int D, bool SCALE>
__device__ __forceinline__ void rope_chunk(uint32_t (&w)[4], int c, const RopeRow& rr, float scale) {
  using C = RopeCfg<D>;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int p0 = 4 * c + 2 * hh, p1 = p0 + 1;  // p0 is even: slot 0 of its unit
    if (C::axis_of(p0) == C::axis_of(p1)) {
      const float4 U = rr.unit(C::axis_of(p0), C::unit_of(p0));
      const uint64_t cc = f2_make(U.x, U.y), ss = f2_make(U.z, U.w);
      const uint64_t a = f2_make(bf16lo_to_f32(w[2 * hh]), bf16lo_to_f32(w[2 * hh + 1]));
      const uint64_t b = f2_make(bf16hi_to_f32(w[2 * hh]), bf16hi_to_f32(w[2 * hh + 1]));
      uint64_t ra = f2_sub(f2_mul(a, cc), f2_mul(b, ss));
      uint64_t rb = f2_fma(a, ss, f2_mul(b, cc));
      if (SCALE) {
        const uint64_t sc = f2_make(scale, scale);
        ra = f2_mul(ra, sc);
        rb = f2_mul(rb, sc);
      }
      float ra0, ra1, rb0, rb1;
      f2_split(ra, ra0, ra1);
      f2_split(rb, rb0, rb1);
      w[2 * hh] = pack_bf16x2(ra0, rb0);
      w[2 * hh + 1] = pack_bf16x2(ra1, rb1);
    } else {
      const float4 U0 = rr.unit(C::axis_of(p0), C::unit_of(p0));
      const float4 U1 = rr.unit(C::axis_of(p1), C::unit_of(p1));
      w[2 * hh] = rot_pair(w[2 * hh], U0.x, U0.z, scale, SCALE);
      w[2 * hh + 1] = rot_pair(w[2 * hh + 1], U1.y, U1.w, scale, SCALE);
    }
  }
}

}  // namespace dev
}  // namespace ckv

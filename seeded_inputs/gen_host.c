/*
 * Seeded synthetic inputs, host side.
 *
 * This module holds no arithmetic of the ConvKV method.  It only produces the
 * bf16 values that both the fp64 oracle and the CUDA path consume, so that the
 * two see bit-identical inputs without either one calling the other.
 *
 * Generator: Philox4x32-10, the counter-based generator of Salmon, Moraes,
 * Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3" (SC'11),
 * written here from its published definition (two 32x32->64 multiplies per
 * round, Weyl key schedule, ten rounds).
 *
 * Value transform (integer-exact, so host and device agree bit for bit):
 * the four 32-bit output words give twelve 10-bit uniforms u_k in [0, 1023]
 * (bits 0-9, 10-19, 20-29 of each word).  Their sum minus its mean, divided
 * by 1024, is an Irwin-Hall(12) variate: mean 0, variance 1 - 2^-20, support
 * +-6 -- the classic sum-of-twelve-uniforms stand-in for N(0,1).  The result
 * n/1024 is exact in fp32; an optional fp32 scale is applied with one IEEE
 * round-to-nearest multiply; the value is then rounded to bf16
 * (round-to-nearest-even) with integer operations.
 *
 * Addressing: counter = (element, frame, state, tensor), key = (seed, 0).
 */
#include <stdint.h>
#include <string.h>

#define SI_M0 0xD2511F53u
#define SI_M1 0xCD9E8D57u
#define SI_W0 0x9E3779B9u
#define SI_W1 0xBB67AE85u

void si_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
  uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) { k0 += SI_W0; k1 += SI_W1; }
    uint64_t p0 = (uint64_t)SI_M0 * (uint64_t)c0;
    uint64_t p1 = (uint64_t)SI_M1 * (uint64_t)c2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c1 ^ k0;
    uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

static inline uint16_t si_f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

uint16_t si_value_bf16(uint32_t seed, uint32_t tensor, uint32_t state, uint32_t frame,
                       uint32_t elem, float scale) {
  uint32_t ctr[4] = {elem, frame, state, tensor};
  uint32_t key[2] = {seed, 0u};
  uint32_t w[4];
  si_philox4x32_10(ctr, key, w);
  int32_t sum = 0;
  for (int i = 0; i < 4; ++i) {
    sum += (int32_t)(w[i] & 1023u);
    sum += (int32_t)((w[i] >> 10) & 1023u);
    sum += (int32_t)((w[i] >> 20) & 1023u);
  }
  float x = (float)(sum - 6138) * (1.0f / 1024.0f); /* exact: |sum-6138| < 2^13 */
  volatile float xs = x * scale;                    /* one IEEE RN multiply */
  return si_f32_to_bf16_rne(xs);
}

/* out[f * frame_elems + e] = value(seed, tensor, state, frame0 + f, e, scale) */
void si_fill_bf16(uint16_t* out, uint32_t seed, uint32_t tensor, uint32_t state,
                  uint32_t frame0, uint32_t nframes, uint64_t frame_elems, float scale) {
  int64_t total = (int64_t)nframes * (int64_t)frame_elems;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < total; ++i) {
    uint32_t f = (uint32_t)(i / (int64_t)frame_elems);
    uint32_t e = (uint32_t)(i % (int64_t)frame_elems);
    out[i] = si_value_bf16(seed, tensor, state, frame0 + f, e, scale);
  }
}

/* Values at an explicit list of element indices of one frame (used to sample
 * single query rows of very large frames without materialising them). */
void si_fill_bf16_indexed(uint16_t* out, uint32_t seed, uint32_t tensor, uint32_t state,
                          uint32_t frame, const uint32_t* elems, int64_t n, float scale) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = si_value_bf16(seed, tensor, state, frame, elems[i], scale);
}

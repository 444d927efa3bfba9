// Conv compression of evicted frames on the 5th-generation tensor cores.
//
// SoulX-LiveAct blog walk-through, section "ConvKV Memory": old KV is
// compressed by a lightweight 1D convolution into a fixed-length memory; the
// aiboss88.com summary (ConvKV Memory bullet) gives the 5:1 ratio.  Per head h,
// for one group of 5 evicted frames x_0..x_4 (oldest first):
//     out[s, o] = sum_{j<5} sum_{i<D} W[h, o, i, j] * x_j[s, i]
// i.e. one GEMM per (group, K|V, head): [T x 5D] . [5D x D], accumulated in
// fp32 in tensor memory and rounded to bf16 into the memory slot.
//
// One CTA computes a 128-token x D tile: five k-blocks (one per evicted frame),
// each a TMA box of the frame's rows for this head (ring slots may wrap; each
// k-block is its own load, so wrap costs nothing) and the matching D x D
// weight block.  Warp 0 issues TMA, warp 1 issues tcgen05.mma (M=128, N=D,
// K=16 steps) and owns the TMEM accumulator, warps 2-5 drain it.
#include "convkv_internal.h"
#include "sm100.cuh"
#include "nvfp4.cuh"

namespace ckv {
namespace {

using namespace dev;

template <int D>
struct ConvCfg {
  static constexpr int BM = 128;
  static constexpr int STAGES = 3;
  static constexpr int NBOX = D / 64;                // 64-channel (128-byte) boxes per row
  static constexpr int A_BYTES = BM * D * 2;         // token rows x input channels
  static constexpr int B_BYTES = D * D * 2;          // output channels x input channels
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = D < 32 ? 32 : D;
  static constexpr int THREADS = 192;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + 256;
};

template <int D>
__global__ void __launch_bounds__(ConvCfg<D>::THREADS, 1)
    conv_bf16_kernel(const __grid_constant__ CUtensorMap tmRingK, const __grid_constant__ CUtensorMap tmRingV,
                     const __grid_constant__ CUtensorMap tmW, const ConvParams p) {
  using C = ConvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                 // [STAGES]
  uint64_t* empty = bars + C::STAGES;    // [STAGES]
  uint64_t* acc_full = bars + 2 * C::STAGES;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = blockIdx.x, head = blockIdx.y;
  const int kv = blockIdx.z & 1;
  const int sg = blockIdx.z >> 1;
  const int state = sg % p.S;
  const int g = sg / p.S;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const CUtensorMap* ring = kv ? &tmRingV : &tmRingK;
      tma_prefetch_desc(ring);
      tma_prefetch_desc(&tmW);
      int issued[C::STAGES] = {};
      for (int j = 0; j < kEvict; ++j) {
        const int st = j % C::STAGES;
        if (j >= C::STAGES && !mbar_wait(&empty[st], ((j / C::STAGES) - 1) & 1, abort_flag)) break;
        uint8_t* a = stages + st * C::STAGE_BYTES;
        uint8_t* b = a + C::A_BYTES;
        mbar_expect_tx(&full[st], C::STAGE_BYTES);
        const int row = p.grp[g].ring_slot[j] * p.T + mt * C::BM;
        const int wrow = ((kv * p.H + head) * kEvict + j) * D;
#pragma unroll
        for (int bx = 0; bx < C::NBOX; ++bx) {
          tma_load_4d(a + bx * (C::BM * 128), ring, &full[st], bx * 64, head, row, state);
          tma_load_3d(b + bx * (D * 128), &tmW, &full[st], bx * 64, wrow, state);
        }
        ++issued[st];
      }
      // drain: every load issued must have landed before the CTA may exit
      for (int st = 0; st < C::STAGES; ++st) {
        if (issued[st] > 0) {
          volatile int no_abort = 0;
          mbar_wait(&full[st], (issued[st] - 1) & 1, &no_abort);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, D, false, false);
      bool any = false;
      for (int j = 0; j < kEvict; ++j) {
        const int st = j % C::STAGES;
        if (!mbar_wait(&full[st], (j / C::STAGES) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t a = smem_u32(stages + st * C::STAGE_BYTES);
        const uint32_t b = a + C::A_BYTES;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = (ks & 3) * 32;
          const uint64_t ad = sdesc_sw128(a + (ks >> 2) * (C::BM * 128) + koff, 16, 1024);
          const uint64_t bd = sdesc_sw128(b + (ks >> 2) * (D * 128) + koff, 16, 1024);
          mma_ss(tmem, ad, bd, idesc, (j | ks) != 0);
        }
        any = true;
        tc_commit(&empty[st]);
      }
      tc_commit(acc_full);
      if (any) {
        volatile int no_abort = 0;
        tc_commit(drain);
        mbar_wait(drain, 0, &no_abort);
      }
    }
  } else {
    // epilogue: warps 2..5 -> TMEM lanes 32*(warp%4) .. +31
    const int lane_base = (warp & 3) * 32;
    const int r = lane_base + lane;
    const int token = mt * C::BM + r;
    if (mbar_wait_warp(acc_full, 0, abort_flag)) {
      tc_fence_after();
      __nv_bfloat16* dst_base = static_cast<__nv_bfloat16*>(kv ? p.memV : p.memK);
      const int64_t row = (static_cast<int64_t>(state) * p.C + p.grp[g].mem_pos) * p.T + token;
      uint4* dst = reinterpret_cast<uint4*>(dst_base + (row * p.H + head) * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(lane_base) << 16) + c * 32, v);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
        if (token < p.T) {
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[c * 4 + q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicExch(p.status, kStatusTimeout);
}


// ---------------------------------------------------------------------------
// fp8 (e4m3) format.  The evicted frames are e4m3 with one fp32 scale per
// (frame, head); the A operand is dequantised to bf16 (x * scale) in shared
// memory by warps 2-5 instead of TMA.  The slot is stored e4m3 with one scale
// per (slot, head) = amax / 448 over the slot's [T, D] values, so the launch
// runs twice: pass 1 only reduces amax (atomicMax on the fp32 bit pattern,
// values are non-negative), pass 2 recomputes the same tiles and quantises
// with that scale (round-to-nearest-even, saturating to +-448).  FMT 2 is the
// NVFP4 format: e2m1 codes with an e4m3 scale per 16 channels and the fp32
// scale per (frame or slot, head) of the same two-pass rule (nvfp4.cuh).
__device__ __forceinline__ void e4m3x2_to_f32_c(uint32_t two, float& lo, float& hi) {
  uint32_t h2;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h2) : "r"(two));
  lo = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
  hi = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
}
// two fp32 -> two e4m3 codes, lo in the low byte
__device__ __forceinline__ uint32_t f32x2_to_e4m3(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int D, int PASS, int FMT>
__global__ void __launch_bounds__(ConvCfg<D>::THREADS, 1)
    conv_lowp_kernel(const __grid_constant__ CUtensorMap tmW, const ConvParams p) {
  using C = ConvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::STAGES * C::STAGE_BYTES);
  uint64_t* b_full = bars;                    // [STAGES] weights landed (TMA)
  uint64_t* a_full = bars + C::STAGES;        // [STAGES] A dequantised (128 threads)
  uint64_t* empty = bars + 2 * C::STAGES;     // [STAGES]
  uint64_t* acc_full = bars + 3 * C::STAGES;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  unsigned int* red = reinterpret_cast<unsigned int*>(tmem_slot + 2);  // CTA amax

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = blockIdx.x, head = blockIdx.y;
  const int kv = blockIdx.z & 1;
  const int sg = blockIdx.z >> 1;
  const int state = sg % p.S;
  const int g = sg / p.S;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&a_full[i], 128);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    *red = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmW);
      int issued[C::STAGES] = {};
      for (int j = 0; j < kEvict; ++j) {
        const int st = j % C::STAGES;
        if (j >= C::STAGES && !mbar_wait(&empty[st], ((j / C::STAGES) - 1) & 1, abort_flag)) break;
        uint8_t* b = stages + st * C::STAGE_BYTES + C::A_BYTES;
        mbar_expect_tx(&b_full[st], C::B_BYTES);
        const int wrow = ((kv * p.H + head) * kEvict + j) * D;
#pragma unroll
        for (int bx = 0; bx < C::NBOX; ++bx) tma_load_3d(b + bx * (D * 128), &tmW, &b_full[st], bx * 64, wrow, state);
        ++issued[st];
      }
      volatile int no_abort = 0;
      for (int st = 0; st < C::STAGES; ++st)
        if (issued[st] > 0) mbar_wait(&b_full[st], (issued[st] - 1) & 1, &no_abort);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, D, false, false);
      bool any = false;
      for (int j = 0; j < kEvict; ++j) {
        const int st = j % C::STAGES;
        if (!mbar_wait(&a_full[st], (j / C::STAGES) & 1, abort_flag)) break;
        if (!mbar_wait(&b_full[st], (j / C::STAGES) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t a = smem_u32(stages + st * C::STAGE_BYTES);
        const uint32_t b = a + C::A_BYTES;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = (ks & 3) * 32;
          const uint64_t ad = sdesc_sw128(a + (ks >> 2) * (C::BM * 128) + koff, 16, 1024);
          const uint64_t bd = sdesc_sw128(b + (ks >> 2) * (D * 128) + koff, 16, 1024);
          mma_ss(tmem, ad, bd, idesc, (j | ks) != 0);
        }
        any = true;
        tc_commit(&empty[st]);
      }
      tc_commit(acc_full);
      if (any) {
        volatile int no_abort = 0;
        tc_commit(drain);
        mbar_wait(drain, 0, &no_abort);
      }
    }
  } else {
    // warps 2..5: dequantise A (one token row per thread), then drain the accumulator
    const int lane_base = (warp & 3) * 32;
    const int r = lane_base + lane;
    const int token = mt * C::BM + r;
    const bool valid = token < p.T;
    bool alive = true;
    for (int j = 0; j < kEvict; ++j) {
      const int st = j % C::STAGES;
      if (j >= C::STAGES && !mbar_wait(&empty[st], ((j / C::STAGES) - 1) & 1, abort_flag)) {
        alive = false;
        break;
      }
      const int slot = p.grp[g].ring_slot[j];
      const float sc = __ldg(&p.ring_scale[((static_cast<int64_t>(state) * 2 + kv) * p.R + slot) * p.H + head]);
      const int64_t grow = (static_cast<int64_t>(state) * p.R * p.T + static_cast<int64_t>(slot) * p.T + token) * p.H + head;
      uint8_t* rowp = stages + st * C::STAGE_BYTES + r * 128;
      const int sw = r & 7;
      if (FMT == 2) {
        // e2m1 pairs: 4 bytes per 8 channels, one e4m3 block scale per 16 channels
        const uint32_t* src = reinterpret_cast<const uint32_t*>(p.ring8[kv] + grow * (D / 2));
        const uint8_t* bs = p.ring_bs[kv] + grow * (D / 16);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          uint32_t o[4] = {0, 0, 0, 0};
          if (valid) {
            const float e_b = __fmul_rn(fp4::e4m3_to_f32(__ldg(bs + (c >> 1))), sc);
            fp4::decode8(__ldg(src + c), e_b, o);
          }
          *reinterpret_cast<uint4*>(rowp + (c >> 3) * (C::BM * 128) + (((c & 7) ^ sw) << 4)) =
              make_uint4(o[0], o[1], o[2], o[3]);
        }
      } else {
      const uint8_t* src = p.ring8[kv] + grow * D;
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint4 raw = valid ? __ldg(reinterpret_cast<const uint4*>(src) + k) : make_uint4(0, 0, 0, 0);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int c = 2 * k + u;
          uint32_t o[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t word = w[2 * u + (q >> 1)];
            float a, b;
            e4m3x2_to_f32_c((q & 1) ? (word >> 16) : (word & 0xFFFFu), a, b);
            o[q] = pack_bf16x2(a * sc, b * sc);
          }
          *reinterpret_cast<uint4*>(rowp + (c >> 3) * (C::BM * 128) + (((c & 7) ^ sw) << 4)) =
              make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      }
      fence_proxy_async_smem();
      mbar_arrive(&a_full[st]);
    }
    if (alive && mbar_wait_warp(acc_full, 0, abort_flag)) {
      tc_fence_after();
      const int64_t aidx = ((static_cast<int64_t>(state) * 2 + kv) * p.ngroups + g) * p.H + head;
      if (PASS == 1) {
        float mx = 0.0f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + (static_cast<uint32_t>(lane_base) << 16) + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) mx = fmaxf(mx, fabsf(__uint_as_float(v[e])));
        }
        if (!valid) mx = 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) atomicMax(red, __float_as_uint(mx));
      } else if (FMT == 2) {
        const float gs = fp4::tensor_scale(__uint_as_float(p.amax[aidx]));
        const int64_t row = ((static_cast<int64_t>(state) * p.C + p.grp[g].mem_pos) * p.T + token) * p.H + head;
        uint2* dst = reinterpret_cast<uint2*>(static_cast<uint8_t*>(kv ? p.memV : p.memK) + row * (D / 2));
        uint8_t* bs = p.mem_bs[kv] + row * (D / 16);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + (static_cast<uint32_t>(lane_base) << 16) + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            float xs[fp4::kBlock];
            float a_b = 0.0f;
#pragma unroll
            for (int e = 0; e < fp4::kBlock; ++e) {
              xs[e] = __uint_as_float(v[hb * 16 + e]);
              a_b = fmaxf(a_b, fabsf(xs[e]));
            }
            float e_b;
            const uint32_t sc = fp4::block_scale(a_b, gs, e_b);
            const uint2 cw = fp4::encode_block(xs, e_b);
            if (valid) {
              dst[2 * c + hb] = cw;
              bs[2 * c + hb] = static_cast<uint8_t>(sc);
            }
          }
        }
        if (mt == 0 && r == 0)
          p.mem_scale[((static_cast<int64_t>(state) * 2 + kv) * p.C + p.grp[g].mem_pos) * p.H + head] = gs;
      } else {
        const float amax = __uint_as_float(p.amax[aidx]);
        const float scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        uint8_t* dst = static_cast<uint8_t*>(kv ? p.memV : p.memK) +
                       (((static_cast<int64_t>(state) * p.C + p.grp[g].mem_pos) * p.T + token) * p.H + head) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + (static_cast<uint32_t>(lane_base) << 16) + c * 32, v);
          tmem_ld_wait();
          uint32_t w[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t lo = f32x2_to_e4m3(__fdiv_rn(__uint_as_float(v[4 * e]), scale),
                                              __fdiv_rn(__uint_as_float(v[4 * e + 1]), scale));
            const uint32_t hi = f32x2_to_e4m3(__fdiv_rn(__uint_as_float(v[4 * e + 2]), scale),
                                              __fdiv_rn(__uint_as_float(v[4 * e + 3]), scale));
            w[e] = lo | (hi << 16);
          }
          if (valid) {
            reinterpret_cast<uint4*>(dst)[2 * c] = make_uint4(w[0], w[1], w[2], w[3]);
            reinterpret_cast<uint4*>(dst)[2 * c + 1] = make_uint4(w[4], w[5], w[6], w[7]);
          }
        }
        if (mt == 0 && r == 0)
          p.mem_scale[((static_cast<int64_t>(state) * 2 + kv) * p.C + p.grp[g].mem_pos) * p.H + head] = scale;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (PASS == 1 && threadIdx.x == 64 && *red != 0) {
    const int64_t aidx = ((static_cast<int64_t>(state) * 2 + kv) * p.ngroups + g) * p.H + head;
    atomicMax(&p.amax[aidx], *red);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicExch(p.status, kStatusTimeout);
}

}  // namespace

namespace {

template <int D, int FMT>
int launch_lowp(const ConvParams& p, const CUtensorMap& wmap, cudaStream_t s) {
  using C = ConvCfg<D>;
  dim3 grid((p.T + 127) / 128, p.H, p.ngroups * p.S * 2);
  auto k1 = conv_lowp_kernel<D, 1, FMT>;
  auto k2 = conv_lowp_kernel<D, 2, FMT>;
  cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  k1<<<grid, C::THREADS, C::SMEM, s>>>(wmap, p);
  k2<<<grid, C::THREADS, C::SMEM, s>>>(wmap, p);
  return static_cast<int>(cudaGetLastError());
}

template <int FMT>
int launch_lowp_d(int D, const ConvParams& p, const CUtensorMap& wmap, cudaStream_t s) {
  if (p.ngroups <= 0) return 0;
  cudaError_t e = cudaMemsetAsync(p.amax, 0, sizeof(unsigned int) * p.S * 2 * p.ngroups * p.H, s);
  if (e != cudaSuccess) return static_cast<int>(e);
  if (D == 128) return launch_lowp<128, FMT>(p, wmap, s);
  if (D == 64) return launch_lowp<64, FMT>(p, wmap, s);
  return static_cast<int>(cudaErrorInvalidValue);
}

}  // namespace

int launch_conv_fp8(int D, const ConvParams& p, const CUtensorMap& wmap, cudaStream_t s) {
  return launch_lowp_d<1>(D, p, wmap, s);
}

int launch_conv_fp4(int D, const ConvParams& p, const CUtensorMap& wmap, cudaStream_t s) {
  return launch_lowp_d<2>(D, p, wmap, s);
}


size_t conv_smem_bytes(int D) { return D == 128 ? ConvCfg<128>::SMEM : ConvCfg<64>::SMEM; }

int launch_conv_bf16(int D, const ConvParams& p, const CUtensorMap& ringK, const CUtensorMap& ringV,
                     const CUtensorMap& wmap, cudaStream_t s) {
  if (p.ngroups <= 0) return 0;
  dim3 grid((p.T + 127) / 128, p.H, p.ngroups * p.S * 2);
  if (D == 128) {
    auto k = conv_bf16_kernel<128>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ConvCfg<128>::SMEM);
    k<<<grid, ConvCfg<128>::THREADS, ConvCfg<128>::SMEM, s>>>(ringK, ringV, wmap, p);
  } else if (D == 64) {
    auto k = conv_bf16_kernel<64>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ConvCfg<64>::SMEM);
    k<<<grid, ConvCfg<64>::THREADS, ConvCfg<64>::SMEM, s>>>(ringK, ringV, wmap, p);
  } else {
    return static_cast<int>(cudaErrorInvalidValue);
  }
  return static_cast<int>(cudaGetLastError());
}

}  // namespace ckv

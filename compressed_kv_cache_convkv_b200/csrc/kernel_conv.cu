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
// One work unit is a 128-token x D tile: five k-blocks (one per evicted frame),
// each a TMA box of the frame's rows for this head (ring slots may wrap; each
// k-block is its own load, so wrap costs nothing) and the matching D x D
// weight block.  Warp 0 issues TMA, warp 1 issues tcgen05.mma (M=128, N=D,
// K=16 steps) and owns the TMEM accumulators, warps 2-5 drain them.  The bf16
// and low-precision kernels are persistent (one CTA per SM walking the units).
#include "convkv_internal.h"
#include "sm100.cuh"
#include "nvfp4.cuh"
#include "quant_div.cuh"
#include "token_walk.h"

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

// One work unit = (128-token tile mt, head, K|V, state, group); units are numbered
// with mt fastest, so consecutive units of a CTA share the head's weights in L2.
struct ConvUnit {
  int mt, head, kv, state, g;
};
__device__ __forceinline__ ConvUnit conv_unit(int u, int MT, const ConvParams& p) {
  ConvUnit c;
  c.mt = u % MT;
  int rest = u / MT;
  c.head = rest % p.H;
  rest /= p.H;
  c.kv = rest & 1;
  const int sg = rest >> 1;
  c.state = sg % p.S;
  c.g = sg / p.S;
  return c;
}

// Persistent: each CTA walks units blockIdx.x, blockIdx.x + gridDim.x, ...  The
// producer streams the units' k-blocks through a 3-stage ring without pausing
// between units; the accumulator is double-buffered in TMEM, so the epilogue of one
// unit overlaps the loads and MMAs of the next.
template <int D>
__global__ void __launch_bounds__(ConvCfg<D>::THREADS, 1)
    conv_bf16_kernel(const __grid_constant__ CUtensorMap tmRingK, const __grid_constant__ CUtensorMap tmRingV,
                     const __grid_constant__ CUtensorMap tmW, const ConvParams p, int MT, int units) {
  using C = ConvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                    // [STAGES]
  uint64_t* empty = bars + C::STAGES;       // [STAGES]
  uint64_t* acc_full = bars + 2 * C::STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmRingK);
      tma_prefetch_desc(&tmRingV);
      tma_prefetch_desc(&tmW);
      int issued[C::STAGES] = {};
      int it = 0;  // k-blocks issued by this CTA
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const ConvUnit cu = conv_unit(u, MT, p);
        const CUtensorMap* ring = cu.kv ? &tmRingV : &tmRingK;
        for (int j = 0; j < kEvict; ++j, ++it) {
          const int st = it % C::STAGES;
          if (it >= C::STAGES && !mbar_wait(&empty[st], ((it / C::STAGES) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* a = stages + st * C::STAGE_BYTES;
          uint8_t* b = a + C::A_BYTES;
          mbar_expect_tx(&full[st], C::STAGE_BYTES);
          const int row = p.grp[cu.g].ring_slot[j] * p.T + cu.mt * C::BM;
          const int wrow = ((cu.kv * p.H + cu.head) * kEvict + j) * D;
#pragma unroll
          for (int bx = 0; bx < C::NBOX; ++bx) {
            tma_load_4d(a + bx * (C::BM * 128), ring, &full[st], bx * 64, cu.head, row, cu.state);
            tma_load_3d(b + bx * (D * 128), &tmW, &full[st], bx * 64, wrow, cu.state);
          }
          ++issued[st];
        }
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
      bool any = false, ok = true;
      int it = 0, n = 0;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++n) {
        const int ab = n & 1;
        if (n >= 2 && !mbar_wait(&acc_empty[ab], ((n >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t acc = tmem + ab * C::TMEM_COLS;
        for (int j = 0; j < kEvict; ++j, ++it) {
          const int st = it % C::STAGES;
          if (!mbar_wait(&full[st], (it / C::STAGES) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(stages + st * C::STAGE_BYTES);
          const uint32_t b = a + C::A_BYTES;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t koff = (ks & 3) * 32;
            const uint64_t ad = sdesc_sw128(a + (ks >> 2) * (C::BM * 128) + koff, 16, 1024);
            const uint64_t bd = sdesc_sw128(b + (ks >> 2) * (D * 128) + koff, 16, 1024);
            mma_ss(acc, ad, bd, idesc, (j | ks) != 0);
          }
          any = true;
          tc_commit(&empty[st]);
        }
        if (ok) tc_commit(&acc_full[ab]);
      }
      if (any) {
        volatile int no_abort = 0;
        tc_commit(drain);
        mbar_wait(drain, 0, &no_abort);
      }
    }
  } else {
    // epilogue: warps 2..5 -> TMEM lanes 32*(warp%4) .. +31, one token row each
    const int lane_base = (warp & 3) * 32;
    const int r = lane_base + lane;
    int n = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++n) {
      const int ab = n & 1;
      if (!mbar_wait_warp(&acc_full[ab], (n >> 1) & 1, abort_flag)) break;
      tc_fence_after();
      const ConvUnit cu = conv_unit(u, MT, p);
      const int token = cu.mt * C::BM + r;
      __nv_bfloat16* dst_base = static_cast<__nv_bfloat16*>(cu.kv ? p.memV : p.memK);
      const int64_t row = (static_cast<int64_t>(cu.state) * p.C + p.grp[cu.g].mem_pos) * p.T + token;
      uint4* dst = reinterpret_cast<uint4*>(dst_base + (row * p.H + cu.head) * D);
      const uint32_t tacc = tmem + ab * C::TMEM_COLS + (static_cast<uint32_t>(lane_base) << 16);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tacc + c * 32, v);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
        if (token < p.T) {
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[c * 4 + q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
      }
      // the accumulator may be overwritten once every row of it has been read
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * C::TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicExch(p.status, kStatusTimeout);
}


// ---------------------------------------------------------------------------
// fp8 (e4m3) format.  The evicted frames are e4m3 with one fp32 scale per
// (frame, head); the A operand's codes arrive by TMA and are dequantised to bf16
// (x * scale) in shared memory by warps 6-13.  The slot is stored e4m3 with one scale
// per (slot, head) = amax / 448 over the slot's [T, D] values, so the conv keeps
// its fp32 outputs in a scratch and reduces amax (atomicMax on the fp32 bit
// pattern, values are non-negative); slot_quant_kernel then quantises them with
// that scale (round-to-nearest-even, saturating to +-448).  FMT 2 is the NVFP4
// format: e2m1 codes with an e4m3 scale per 16 channels and the fp32 scale per
// (frame or slot, head) from the same amax (nvfp4.cuh).
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

// Low-precision A operand: the evicted frame's code tile (128 token rows of CB code
// bytes of one head) is staged by TMA into the upper half of the A stage, with the
// CB-byte swizzle, and expanded in place into the bf16 tile by warps 6-13 (two
// threads per row, half a row each; a row's output covers other rows' codes, so the
// threads read all their codes and meet at a barrier before writing).
template <int D, int FMT>
struct LowpA {
  static constexpr int CB = FMT == 2 ? D / 2 : D;
  static constexpr int BYTES = 128 * CB;
  static constexpr int OFF = ConvCfg<D>::A_BYTES / 2;
  static constexpr int NCH = CB / 16;
  static constexpr uint32_t MASK = CB == 128 ? 7u : (CB == 64 ? 3u : 1u);
};

__device__ __forceinline__ bool conv_bar_all(int id, int nthreads, bool v) {
  uint32_t r;
  __syncwarp();
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

template <int D>
struct LowpCfg {
  static constexpr int THREADS = 448;  // producer, MMA, 4 epilogue warps, 8 converter warps
};

// Persistent like the bf16 kernel: CTAs walk the units, the accumulator is double-
// buffered in TMEM.  The epilogue keeps the fp32 outputs (p.acc) and reduces each new
// slot's amax over its tokens; slot_quant_kernel then quantises them with it.
template <int D, int FMT>
__global__ void __launch_bounds__(LowpCfg<D>::THREADS, 1)
    conv_lowp_kernel(const __grid_constant__ CUtensorMap tmCodesK, const __grid_constant__ CUtensorMap tmCodesV,
                     const __grid_constant__ CUtensorMap tmW, const ConvParams p, int MT, int units) {
  using C = ConvCfg<D>;
  using LA = LowpA<D, FMT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                       // [STAGES] codes + weights landed (TMA)
  uint64_t* a_ready = bars + C::STAGES;        // [STAGES] A expanded to bf16 (128 threads)
  uint64_t* empty = bars + 2 * C::STAGES;      // [STAGES]
  uint64_t* acc_full = bars + 3 * C::STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&a_ready[i], 256);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmCodesK);
      tma_prefetch_desc(&tmCodesV);
      tma_prefetch_desc(&tmW);
      int issued[C::STAGES] = {};
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const ConvUnit cu = conv_unit(u, MT, p);
        const CUtensorMap* codes = cu.kv ? &tmCodesV : &tmCodesK;
        for (int j = 0; j < kEvict; ++j, ++it) {
          const int st = it % C::STAGES;
          if (it >= C::STAGES && !mbar_wait(&empty[st], ((it / C::STAGES) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* a = stages + st * C::STAGE_BYTES;
          uint8_t* b = a + C::A_BYTES;
          mbar_expect_tx(&full[st], LA::BYTES + C::B_BYTES);
          const int row = p.grp[cu.g].ring_slot[j] * p.T + cu.mt * C::BM;
          tma_load_4d(a + LA::OFF, codes, &full[st], 0, cu.head, row, cu.state);
          const int wrow = ((cu.kv * p.H + cu.head) * kEvict + j) * D;
#pragma unroll
          for (int bx = 0; bx < C::NBOX; ++bx) tma_load_3d(b + bx * (D * 128), &tmW, &full[st], bx * 64, wrow, cu.state);
          ++issued[st];
        }
      }
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
      bool any = false, ok = true;
      int it = 0, n = 0;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++n) {
        const int ab = n & 1;
        if (n >= 2 && !mbar_wait(&acc_empty[ab], ((n >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t acc = tmem + ab * C::TMEM_COLS;
        for (int j = 0; j < kEvict; ++j, ++it) {
          const int st = it % C::STAGES;
          // the weights' TMA (full) and the expanded A (a_ready) of the stage
          if (!mbar_wait(&full[st], (it / C::STAGES) & 1, abort_flag) ||
              !mbar_wait(&a_ready[st], (it / C::STAGES) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(stages + st * C::STAGE_BYTES);
          const uint32_t b = a + C::A_BYTES;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t koff = (ks & 3) * 32;
            const uint64_t ad = sdesc_sw128(a + (ks >> 2) * (C::BM * 128) + koff, 16, 1024);
            const uint64_t bd = sdesc_sw128(b + (ks >> 2) * (D * 128) + koff, 16, 1024);
            mma_ss(acc, ad, bd, idesc, (j | ks) != 0);
          }
          any = true;
          tc_commit(&empty[st]);
        }
        if (ok) tc_commit(&acc_full[ab]);
      }
      if (any) {
        volatile int no_abort = 0;
        tc_commit(drain);
        mbar_wait(drain, 0, &no_abort);
      }
    }
  } else if (warp >= 6) {
    // warps 6..13: expand each staged code tile to bf16 rows (bf16(fp32(code * scale))).
    // Two threads per token row, one half of its channels each; all codes of the tile
    // are read before any row is written (a row's output covers other threads' codes),
    // and the barrier also carries a timeout anywhere in the group to all of it.
    constexpr int HALF_CH = LA::NCH / 2;              // 16-byte code chunks per half row
    constexpr int HALF_C = D / 16;                    // 8-channel output chunks per half row
    const int t = threadIdx.x - 192;
    const int r = t & 127, hf = t >> 7;
    int it = 0;
    bool live = true;
    for (int u = blockIdx.x; u < units && live; u += gridDim.x) {
      const ConvUnit cu = conv_unit(u, MT, p);
      const int token = cu.mt * C::BM + r;
      const bool valid = token < p.T;
      for (int j = 0; j < kEvict; ++j, ++it) {
        const int st = it % C::STAGES;
        bool ok = mbar_wait(&full[st], (it / C::STAGES) & 1, abort_flag);
        uint8_t* a = stages + st * C::STAGE_BYTES;
        const int slot = p.grp[cu.g].ring_slot[j];
        const float sc = __ldg(&p.ring_scale[((static_cast<int64_t>(cu.state) * 2 + cu.kv) * p.R + slot) * p.H + cu.head]);
        const int64_t grow =
            (static_cast<int64_t>(cu.state) * p.R * p.T + static_cast<int64_t>(slot) * p.T + token) * p.H + cu.head;
        uint4 raw[HALF_CH];
        uint32_t bsw = 0;
        if (ok) {
#pragma unroll
          for (int k = 0; k < HALF_CH; ++k) {
            const uint32_t logical = static_cast<uint32_t>(r * LA::CB + (hf * HALF_CH + k) * 16);
            const uint32_t phys = logical ^ (((logical >> 7) & LA::MASK) << 4);
            raw[k] = valid ? *reinterpret_cast<const uint4*>(a + LA::OFF + phys) : make_uint4(0, 0, 0, 0);
          }
          if constexpr (FMT == 2) {
            // this half's D/32 block scales (4 bytes at D = 128, 2 at D = 64)
            const uint8_t* bs = p.ring_bs[cu.kv] + grow * (D / 16) + hf * (D / 32);
#pragma unroll
            for (int k = 0; k < D / 32; ++k) bsw |= valid ? static_cast<uint32_t>(__ldg(bs + k)) << (8 * k) : 0u;
          }
        }
        ok = conv_bar_all(1, 256, ok);
        if (!ok) {
          live = false;
          break;
        }
        uint8_t* rowp = a + r * 128;
        const int sw = r & 7;
#pragma unroll
        for (int cc = 0; cc < HALF_C; ++cc) {
          const int c = hf * HALF_C + cc;  // 8-channel chunk of the row
          uint32_t o[4];
          if constexpr (FMT == 2) {
            const uint4 r4 = raw[cc >> 2];
            const uint32_t word = (cc & 3) == 0 ? r4.x : ((cc & 3) == 1 ? r4.y : ((cc & 3) == 2 ? r4.z : r4.w));
            const float e_b = __fmul_rn(fp4::e4m3_to_f32(bsw >> (8 * (cc >> 1))), sc);
            fp4::decode8(word, e_b, o);
          } else {
            const uint4 r4 = raw[cc >> 1];
            const uint32_t w0 = (cc & 1) ? r4.z : r4.x, w1 = (cc & 1) ? r4.w : r4.y;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float x0, x1;
              e4m3x2_to_f32_c(((q < 2 ? w0 : w1) >> (16 * (q & 1))) & 0xFFFFu, x0, x1);
              o[q] = pack_bf16x2(x0 * sc, x1 * sc);
            }
          }
          *reinterpret_cast<uint4*>(rowp + (c >> 3) * (C::BM * 128) + (((c & 7) ^ sw) << 4)) =
              make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(&a_ready[st]);
      }
    }
  } else {
    // warps 2..5: drain the accumulator -> fp32 outputs and the slot's amax
    const int lane_base = (warp & 3) * 32;
    const int r = lane_base + lane;
    int n = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++n) {
      const int ab = n & 1;
      if (!mbar_wait_warp(&acc_full[ab], (n >> 1) & 1, abort_flag)) break;
      tc_fence_after();
      const ConvUnit cu = conv_unit(u, MT, p);
      const int token = cu.mt * C::BM + r;
      const bool valid = token < p.T;
      const uint32_t tacc = tmem + ab * C::TMEM_COLS + (static_cast<uint32_t>(lane_base) << 16);
      const int64_t aidx = ((static_cast<int64_t>(cu.state) * 2 + cu.kv) * p.ngroups + cu.g) * p.H + cu.head;
      // amax of the slot, and the fp32 outputs for the quantiser (one row per thread)
      float* orow = p.acc + ((((static_cast<int64_t>(cu.state) * p.ngroups + cu.g) * 2 + cu.kv) * p.T + token) * p.H +
                             cu.head) * D;
      float mx = 0.0f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tacc + c * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) mx = fmaxf(mx, fabsf(__uint_as_float(v[e])));
        if (valid) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            reinterpret_cast<uint4*>(orow + c * 32)[q] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      }
      if (!valid) mx = 0.0f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0 && mx > 0.0f) atomicMax(&p.amax[aidx], __float_as_uint(mx));
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * C::TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicExch(p.status, kStatusTimeout);
}

}  // namespace

namespace {

// Quantisation of the new memory slots from the conv pass's fp32 outputs, with the
// slot's amax from that pass: the same arithmetic as quantising in the conv's
// epilogue (scale = amax / 448, code = e4m3(x / scale); NVFP4: tensor scale, block
// scales, e2m1 codes), so the codes do not depend on which kernel makes them.
// grid = (walkers * slabs, S * ngroups, 2 (K|V)), token walk: each thread owns one
// (head, 8-channel chunk) column (e4m3) or one (head, 16-channel block) column
// (NVFP4) of the slot.
template <int D, int FMT>
__global__ void slot_quant_kernel(ConvParams p) {
  constexpr int CW = FMT == 2 ? fp4::kBlock : 8;          // channels per column
  constexpr int NCOL = D / CW;
  const int cols = p.H * NCOL;
  const int sg = blockIdx.y;
  const int s = sg / p.ngroups;
  const int g = sg - s * p.ngroups;
  const int kv = blockIdx.z;
  const int slabs = (cols + blockDim.x - 1) / blockDim.x;
  const int walker = blockIdx.x / slabs, walkers = gridDim.x / slabs;
  const int col = (blockIdx.x - walker * slabs) * blockDim.x + threadIdx.x;
  if (col >= cols) return;
  const int h = col / NCOL;
  const int c = col - h * NCOL;
  const int64_t aidx = ((static_cast<int64_t>(s) * 2 + kv) * p.ngroups + g) * p.H + h;
  const float amax = __uint_as_float(p.amax[aidx]);
  const int pos = p.grp[g].mem_pos;
  const float* src = p.acc + (((static_cast<int64_t>(s) * p.ngroups + g) * 2 + kv) * p.T) * p.H * D + h * D + c * CW;
  const int64_t row0 = (static_cast<int64_t>(s) * p.C + pos) * p.T * p.H + h;   // token 0's token-head row
  uint8_t* mem = static_cast<uint8_t*>(kv ? p.memV : p.memK);
  if constexpr (FMT == 2) {
    const float gs = fp4::tensor_scale(amax);
    const SharedDivisor g6 = fp4::block_divisor(gs);
    if (walker == 0 && c == 0) p.mem_scale[((static_cast<int64_t>(s) * 2 + kv) * p.C + pos) * p.H + h] = gs;
    for (int tok = walker; tok < p.T; tok += walkers) {
      const float4* x4 = reinterpret_cast<const float4*>(src + static_cast<int64_t>(tok) * p.H * D);
      float xs[fp4::kBlock];
      float a_b = 0.0f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 v = __ldcs(x4 + q);
        xs[4 * q] = v.x;
        xs[4 * q + 1] = v.y;
        xs[4 * q + 2] = v.z;
        xs[4 * q + 3] = v.w;
      }
#pragma unroll
      for (int e = 0; e < fp4::kBlock; ++e) a_b = fmaxf(a_b, fabsf(xs[e]));
      float e_b;
      const uint32_t sc = fp4::block_scale(a_b, gs, g6, e_b);
      const int64_t row = row0 + static_cast<int64_t>(tok) * p.H;
      reinterpret_cast<uint2*>(mem)[row * NCOL + c] = fp4::encode_block(xs, e_b);
      p.mem_bs[kv][row * NCOL + c] = static_cast<uint8_t>(sc);
    }
  } else {
    const float scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    const SharedDivisor dv = make_divisor(scale);
    if (walker == 0 && c == 0) p.mem_scale[((static_cast<int64_t>(s) * 2 + kv) * p.C + pos) * p.H + h] = scale;
    for (int tok = walker; tok < p.T; tok += walkers) {
      const float4* x4 = reinterpret_cast<const float4*>(src + static_cast<int64_t>(tok) * p.H * D);
      const float4 a = __ldcs(x4), b = __ldcs(x4 + 1);
      const uint32_t w0 = f32x2_to_e4m3(div_rn(a.x, dv), div_rn(a.y, dv)) |
                          (f32x2_to_e4m3(div_rn(a.z, dv), div_rn(a.w, dv)) << 16);
      const uint32_t w1 = f32x2_to_e4m3(div_rn(b.x, dv), div_rn(b.y, dv)) |
                          (f32x2_to_e4m3(div_rn(b.z, dv), div_rn(b.w, dv)) << 16);
      const int64_t row = row0 + static_cast<int64_t>(tok) * p.H;
      reinterpret_cast<uint2*>(mem + row * D)[c] = make_uint2(w0, w1);
    }
  }
}

template <int D, int FMT>
int launch_lowp(const ConvParams& p, const CUtensorMap& codesK, const CUtensorMap& codesV, const CUtensorMap& wmap,
                cudaStream_t s) {
  using C = ConvCfg<D>;
  const int MT = (p.T + 127) / 128;
  const int64_t units64 = static_cast<int64_t>(MT) * p.H * 2 * p.S * p.ngroups;
  if (units64 > (int64_t(1) << 30)) return static_cast<int>(cudaErrorInvalidValue);
  const int units = static_cast<int>(units64);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = units < sms ? units : sms;
  auto k1 = conv_lowp_kernel<D, FMT>;
  cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  k1<<<grid, LowpCfg<D>::THREADS, C::SMEM, s>>>(codesK, codesV, wmap, p, MT, units);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return static_cast<int>(e);
  constexpr int NCOL = D / (FMT == 2 ? fp4::kBlock : 8);
  dim3 qgrid(token_grid_x(p.T, p.H * NCOL, 2 * p.S * p.ngroups), p.S * p.ngroups, 2);
  slot_quant_kernel<D, FMT><<<qgrid, kTokenThreads, 0, s>>>(p);
  return static_cast<int>(cudaGetLastError());
}

template <int FMT>
int launch_lowp_d(int D, const ConvParams& p, const CUtensorMap& codesK, const CUtensorMap& codesV,
                  const CUtensorMap& wmap, cudaStream_t s) {
  if (p.ngroups <= 0) return 0;
  cudaError_t e = cudaMemsetAsync(p.amax, 0, sizeof(unsigned int) * p.S * 2 * p.ngroups * p.H, s);
  if (e != cudaSuccess) return static_cast<int>(e);
  if (D == 128) return launch_lowp<128, FMT>(p, codesK, codesV, wmap, s);
  if (D == 64) return launch_lowp<64, FMT>(p, codesK, codesV, wmap, s);
  return static_cast<int>(cudaErrorInvalidValue);
}

}  // namespace

int launch_conv_fp8(int D, const ConvParams& p, const CUtensorMap& codesK, const CUtensorMap& codesV,
                    const CUtensorMap& wmap, cudaStream_t s) {
  return launch_lowp_d<1>(D, p, codesK, codesV, wmap, s);
}

int launch_conv_fp4(int D, const ConvParams& p, const CUtensorMap& codesK, const CUtensorMap& codesV,
                    const CUtensorMap& wmap, cudaStream_t s) {
  return launch_lowp_d<2>(D, p, codesK, codesV, wmap, s);
}


size_t conv_smem_bytes(int D) { return D == 128 ? ConvCfg<128>::SMEM : ConvCfg<64>::SMEM; }

int launch_conv_bf16(int D, const ConvParams& p, const CUtensorMap& ringK, const CUtensorMap& ringV,
                     const CUtensorMap& wmap, cudaStream_t s) {
  if (p.ngroups <= 0) return 0;
  const int MT = (p.T + 127) / 128;
  const int64_t units64 = static_cast<int64_t>(MT) * p.H * 2 * p.S * p.ngroups;
  if (units64 > (int64_t(1) << 30)) return static_cast<int>(cudaErrorInvalidValue);
  const int units = static_cast<int>(units64);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // one persistent CTA per SM (the stage ring takes most of the shared memory)
  const int grid = units < sms ? units : sms;
  if (D == 128) {
    auto k = conv_bf16_kernel<128>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ConvCfg<128>::SMEM);
    k<<<grid, ConvCfg<128>::THREADS, ConvCfg<128>::SMEM, s>>>(ringK, ringV, wmap, p, MT, units);
  } else if (D == 64) {
    auto k = conv_bf16_kernel<64>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ConvCfg<64>::SMEM);
    k<<<grid, ConvCfg<64>::THREADS, ConvCfg<64>::SMEM, s>>>(ringK, ringV, wmap, p, MT, units);
  } else {
    return static_cast<int>(cudaErrorInvalidValue);
  }
  return static_cast<int>(cudaGetLastError());
}

}  // namespace ckv

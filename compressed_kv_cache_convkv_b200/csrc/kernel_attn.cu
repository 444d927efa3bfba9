// Fused reset-RoPE attention of the current block over [memory | window | current].
//
// What it computes (SoulX-LiveAct): for each head and each query row of the
// current block,
//     o = sum_k softmax_k( <R(pos_q) q, R(pos_k) k> / sqrt(D) ) v_k
// over every key of the memory slots, the window frames and the current block,
// with no mask inside that set (blog walk-through, "Neighbor Forcing":
// block-wise causal mask; "ConvKV Memory": the four-partition context), the
// RoPE time index reset to run 0.. over memory, window, current (press
// article and aiboss88.com summary: RoPE Reset).  RoPE is relative, so keys are
// rotated once at their stream positions (moving ones again when their reset
// position moves) and only the queries are rotated here.
//
// CTA = one (state, head, 256 query rows) work unit, 12 warps:
//   warp 0      TMA producer: Q (2 tiles of 128 rows), then K/V tiles of 128
//               keys through 3 (K) and 2 (V) stage rings, per key segment
//   warp 1      tcgen05.mma issuer and TMEM owner: S_i = Q_i K^T (SS form),
//               O_i += P_i V (P read from TMEM, TS form); tiles i = 0, 1 are
//               interleaved so one tile's softmax overlaps the other's MMAs
//   warps 4-7   softmax of query tile 0; warps 8-11 softmax of tile 1: one
//               thread per query row; online softmax in fp32 registers with a
//               lazily rescaled running max (the O rescale is only done when
//               the max grows by more than 2^8); P written back over S as bf16
// Every key arrives stored rotated (window and current keys by the append, memory
// slots and reference frames by the rotation kernel whenever their positions move,
// the low-precision window and memory by the dequantisation), so K tiles go from
// TMA straight to the tensor cores; only the queries are rotated here.
// Every operand is bf16.  The e4m3 / NVFP4 caches are dequantised (and their keys
// rotated) once per attend into a bf16 scratch by kernels_dequant.cu, instead of by
// each of the query-block CTAs that read a tile.  One launch covers a group of
// states (grid z); p.state0 is the group's first state.
// TMEM: S_0 | S_1 | O_0 | O_1 = 128 | 128 | D | D columns of 512.
// Every barrier wait is bounded; on expiry the CTA raises an abort flag, skips
// the remaining work, drains its outstanding copies and MMAs, frees TMEM and
// records CONVKV_ERR_DEVICE_TIMEOUT in the status word.
#include "convkv_internal.h"
#include "sm100.cuh"
#include "rope.cuh"

namespace ckv {
namespace {

using namespace dev;

template <int D>
struct AttnCfg {
  static constexpr int BM = 128, BN = 128, QT = 2, KST = 3, VST = 2;
  static constexpr int NBOX = D / 64;
  static constexpr int TILE = 128 * D * 2;     // bytes of one 128-row bf16 tile
  static constexpr int BOX = 128 * 128;        // bytes of one 128-row x 64-channel box
  // 16-byte RoPE table units per position of each axis
  static constexpr int UT = RopeCfg<D>::UT, UH = RopeCfg<D>::UH, UW = RopeCfg<D>::UW;
  static constexpr int O_COL = 256;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 384;
  // registers per thread after re-balancing: the block launches with 168 x 384 (the
  // most 384 threads can have, 65536 / 384 rounded down to a multiple of 8); the
  // producer/MMA warpgroup gives registers to the two softmax warpgroups, and the
  // split must stay within the launch allocation or an increase waits forever
  // producer / MMA warps 112 and softmax warps 192 registers: both roles without
  // spills (at 96 / 200 the MMA issuer's loop reloaded spilled values from local memory)
  static constexpr int REG_LAUNCH = 168, REG_CTRL = 112, REG_SOFTMAX = 192;
  static_assert(128 * REG_CTRL + 256 * REG_SOFTMAX <= THREADS * REG_LAUNCH,
                "register split must fit the launch allocation");
  static constexpr int NBARS = 1 + 1 + 2 * KST + 2 * VST + 3 * 2 + 1;
  static constexpr size_t FIXED =
      1024 + static_cast<size_t>(QT + KST + VST) * TILE + NBARS * 8 + 16 + kMaxSegs * sizeof(KeySeg);
};

// Walks the attend's key tiles segment by segment (no division, no search).
struct TileCursor {
  int s = 0, jt = 0;
  __device__ __forceinline__ void next(const KeySeg* seg) {
    if (++jt * 128 >= seg[s].nrows) {
      ++s;
      jt = 0;
    }
  }
};

// Rotate one 128-byte-swizzled row of a tile in place: adjacent channel pairs
// (2i, 2i+1) of each axis segment [t | h | w] turn by the tabulated angle.
// The swizzle permutes 16-byte chunks only, and a pair never straddles a
// chunk, so the rotation is independent of it.
template <int D, bool SCALE>
__device__ __forceinline__ void rope_row(uint8_t* tile, int row, const RopeRow& rr, float scale) {
  using C = AttnCfg<D>;
  uint8_t* rowp = tile + row * 128;
  const int sw = row & 7;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    uint4* ptr = reinterpret_cast<uint4*>(rowp + (c >> 3) * C::BOX + (((c & 7) ^ sw) << 4));
    const uint4 v = *ptr;
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
    rope_chunk<D, SCALE>(w, c, rr, scale);
    *ptr = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Copy one bf16 row of D channels from global (or peer) memory into row `row` of a
// 128-byte-swizzled tile, zeros when src is null (rows past the block).
template <int D>
__device__ __forceinline__ void load_row(uint8_t* tile, int row, const __nv_bfloat16* src) {
  using C = AttnCfg<D>;
  uint8_t* rowp = tile + row * 128;
  const int sw = row & 7;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint4 v = src ? __ldg(reinterpret_cast<const uint4*>(src) + c) : make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(rowp + (c >> 3) * C::BOX + (((c & 7) ^ sw) << 4)) = v;
  }
}

template <int D>
__global__ void __launch_bounds__(AttnCfg<D>::THREADS, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK0,
                const __grid_constant__ CUtensorMap tmV0, const __grid_constant__ CUtensorMap tmK1,
                const __grid_constant__ CUtensorMap tmV1, const __grid_constant__ CUtensorMap tmK2,
                const __grid_constant__ CUtensorMap tmV2, const __grid_constant__ CUtensorMap tmK3,
                const __grid_constant__ CUtensorMap tmV3, const AttnParams p) {
  using C = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = sQ + C::QT * C::TILE;
  uint8_t* sV = sK + C::KST * C::TILE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + C::VST * C::TILE);
  uint64_t* q_full = bars;
  uint64_t* q_ready = q_full + 1;
  uint64_t* k_full = q_ready + 1;        // [KST]
  uint64_t* k_empty = k_full + C::KST;   // [KST]
  uint64_t* v_full = k_empty + C::KST;   // [VST]
  uint64_t* v_empty = v_full + C::VST;   // [VST]
  uint64_t* s_full = v_empty + C::VST;   // [2]
  uint64_t* p_full = s_full + 2;         // [2]
  uint64_t* o_full = p_full + 2;         // [2]
  uint64_t* drain = o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  KeySeg* seg = reinterpret_cast<KeySeg*>(tmem_slot + 4);
  // cos/sin tables stay in global memory and are read through the read-only cache
  const float4* tab_t = p.tables;
  const float4* tab_h = tab_t + p.tab_t_rows * C::UT;
  const float4* tab_w = tab_h + p.tab_h_rows * C::UH;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // sl: the state within this launch's group (coordinate of the group-local scratch);
  // state: its index in the handle (queries, outputs, staging, reference frames)
  const int head = p.head0 + blockIdx.y, sl = blockIdx.z, state = sl + p.state0;
  const int q_row0 = blockIdx.x * (C::QT * C::BM);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_ready, 2 * C::BM);
    for (int i = 0; i < C::KST; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < C::VST; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], C::BM);
      mbar_init(&o_full[i], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < kMaxSegs) seg[threadIdx.x] = p.seg[threadIdx.x];
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    regs_dec<C::REG_CTRL>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      auto kmap = [&](int buf) { return buf == 0 ? &tmK0 : (buf == 1 ? &tmK1 : (buf == 2 ? &tmK2 : &tmK3)); };
      auto vmap = [&](int buf) { return buf == 0 ? &tmV0 : (buf == 1 ? &tmV1 : (buf == 2 ? &tmV2 : &tmV3)); };
      if (p.sv.G == 0) {
        // sequence-sharded queries are gathered row by row by the softmax warps instead
        tma_prefetch_desc(&tmQ);
        mbar_expect_tx(q_full, C::QT * C::TILE);
#pragma unroll
        for (int i = 0; i < C::QT; ++i)
#pragma unroll
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_4d(sQ + i * C::TILE + bx * C::BOX, &tmQ, q_full, bx * 64, head, q_row0 + i * C::BM, state);
      }
      int kiss[C::KST] = {}, viss[C::VST] = {};
      TileCursor cur;
      for (int j = 0; j < p.ntiles; ++j, cur.next(seg)) {
        const KeySeg& sg = seg[cur.s];
        const int row = sg.row0 + cur.jt * C::BN;
        const int st = sg.local ? sl : state;   // the scratch holds only this launch's group
        const int ks = j % C::KST;
        if (j >= C::KST && !mbar_wait(&k_empty[ks], ((j / C::KST) - 1) & 1, abort_flag)) break;
        mbar_expect_tx(&k_full[ks], C::TILE);
#pragma unroll
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_load_4d(sK + ks * C::TILE + bx * C::BOX, kmap(sg.buf), &k_full[ks], bx * 64, head, row, st);
        ++kiss[ks];
        const int vs = j % C::VST;
        if (j >= C::VST && !mbar_wait(&v_empty[vs], ((j / C::VST) - 1) & 1, abort_flag)) break;
        mbar_expect_tx(&v_full[vs], C::TILE);
#pragma unroll
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_load_4d(sV + vs * C::TILE + bx * C::BOX, vmap(sg.buf), &v_full[vs], bx * 64, head, row, st);
        ++viss[vs];
      }
      // drain: every issued copy must land before the CTA exits
      volatile int no_abort = 0;
      if (p.sv.G == 0) mbar_wait(q_full, 0, &no_abort);
      for (int i = 0; i < C::KST; ++i)
        if (kiss[i] > 0) mbar_wait(&k_full[i], (kiss[i] - 1) & 1, &no_abort);
      for (int i = 0; i < C::VST; ++i)
        if (viss[i] > 0) mbar_wait(&v_full[i], (viss[i] - 1) & 1, &no_abort);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, C::BN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, false, true);
      // descriptors of the tile bases; stepping along K or between tiles only adds
      // (byte offset >> 4) to the 14-bit start-address field, which cannot overflow
      // inside the CTA's shared memory
      const uint64_t dq = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv = sdesc_sw128(smem_u32(sV), C::BOX, 1024);
      bool issued_any = false;
      auto issue_s = [&](int i, int ks) {
        const uint64_t a = dq + static_cast<uint64_t>((i * C::TILE) >> 4);
        const uint64_t b = dk + static_cast<uint64_t>((ks * C::TILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::BOX + (kk & 3) * 32) >> 4);
          mma_ss(tmem + i * 128, a + off, b + off, idesc_qk, kk > 0);
        }
        issued_any = true;
      };
      auto issue_pv = [&](int i, int vs, bool acc) {
        const uint64_t b = dv + static_cast<uint64_t>((vs * C::TILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          mma_ts(tmem + C::O_COL + i * D, tmem + i * 128 + kk * 8, b + static_cast<uint64_t>((kk * 16 * 128) >> 4),
                 idesc_pv, (acc || kk > 0) ? 1u : 0u);
        }
      };
      uint64_t* kr = k_full;  // K tiles arrive rotated: straight from TMA to the tensor cores
      do {
        if (!mbar_wait(q_ready, 0, abort_flag)) break;
        if (!mbar_wait(&kr[0], 0, abort_flag)) break;
        tc_fence_after();
        issue_s(0, 0);
        tc_commit(&s_full[0]);
        issue_s(1, 0);
        tc_commit(&s_full[1]);
        tc_commit(&k_empty[0]);
        bool ok = true;
        for (int j = 0; j < p.ntiles && ok; ++j) {
          const int vs = j % C::VST;
          if (!mbar_wait(&v_full[vs], (j / C::VST) & 1, abort_flag)) { ok = false; break; }
          const bool has_next = j + 1 < p.ntiles;
          const int ksn = (j + 1) % C::KST;
          for (int i = 0; i < 2; ++i) {
            if (!mbar_wait(&p_full[i], j & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_pv(i, vs, j > 0);
            if (i == 1) tc_commit(&v_empty[vs]);
            if (has_next) {
              if (i == 0) {
                if (!mbar_wait(&kr[ksn], ((j + 1) / C::KST) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
              }
              issue_s(i, ksn);
              tc_commit(&s_full[i]);
              if (i == 1) tc_commit(&k_empty[ksn]);
            }
          }
        }
        if (!ok) break;
        tc_commit(&o_full[0]);
        tc_commit(&o_full[1]);
      } while (false);
      if (issued_any) {
        volatile int no_abort = 0;
        tc_commit(drain);
        mbar_wait(drain, 0, &no_abort);
      }
    }
  }
  } else {
    regs_inc<C::REG_SOFTMAX>();
    // ------------------------------------------------------------ softmax
    const int i = (warp - 4) >> 2;
    const int lane_base = (warp & 3) * 32;
    const int r = lane_base + lane;
    const int qr = q_row0 + i * C::BM + r;
    bool alive = true;
    if (p.sv.G == 0) {
      alive = mbar_wait(q_full, 0, abort_flag);
    } else {
      // the row from the rank whose sequence shard holds it (the all-to-all of q)
      int rk = 0;
      const int64_t off = qr < p.Nq ? shard_elem(p.sv, state, qr, head, D, rk) : 0;
      load_row<D>(sQ + i * C::TILE, r, qr < p.Nq ? p.q_sh[rk] + off : nullptr);
    }
    if (alive && qr < p.Nq) {
      const int f = qr / p.T;
      const int s = qr - f * p.T;
      const int t = p.tq0 + f;
      const int y = s / p.grid_w;
      const int x = s - y * p.grid_w;
      const RopeRow rr{tab_t + t * C::UT, tab_h + y * C::UH, tab_w + x * C::UW};
      rope_row<D, true>(sQ + i * C::TILE, r, rr, p.q_scale);
    }
    fence_proxy_async_smem();
    mbar_arrive(q_ready);

    const uint32_t tS = tmem + (static_cast<uint32_t>(lane_base) << 16) + i * 128;
    const uint32_t tO = tmem + (static_cast<uint32_t>(lane_base) << 16) + C::O_COL + i * D;
    float m_run = -INFINITY, l_run = 0.0f;
    TileCursor cur;
    for (int j = 0; j < p.ntiles; ++j, cur.next(seg)) {
      if (!mbar_wait_warp(&s_full[i], j & 1, abort_flag)) { alive = false; break; }
      tc_fence_after();
      const int valid = min(C::BN, seg[cur.s].nrows - cur.jt * C::BN);
      // the whole 128-column row of S in registers, one TMEM round trip
      uint32_t sv[C::BN];
      tmem_ld64(tS, sv);
      tmem_ld64(tS + 64, sv + 64);
      tmem_ld_wait();
      if (valid < C::BN) {
#pragma unroll
        for (int e = 0; e < C::BN; ++e)
          if (e >= valid) sv[e] = __float_as_uint(-INFINITY);
      }
      // row max: 4 independent chains of 3-input max
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int e = 0; e < C::BN; e += 2)
        mx[(e >> 1) & 3] = max3f(mx[(e >> 1) & 3], __uint_as_float(sv[e]), __uint_as_float(sv[e + 1]));
      const float m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      const float m_new = fmaxf(m_run, m_tile);
      // lazy rescale: keep the running max unless it grows by more than 2^8
      bool rescale = false;
      float corr = 1.0f;
      if (j == 0) {
        m_run = m_new;
      } else {
        const bool need = m_new > m_run + 8.0f;
        rescale = __any_sync(0xffffffffu, need);
        if (need) {
          corr = fast_exp2(m_run - m_new);
          l_run *= corr;
          m_run = m_new;
        }
      }
      // P = exp2(S - m) as bf16 pairs, written over the first half of S's columns in two
      // halves; pairs of columns go through the packed fp32x2 add (S - m and row sum)
      const uint64_t neg_m = f2_make(-m_run, -m_run);
      uint64_t lsum[4] = {0, 0, 0, 0};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // packed pair e of this half lands in sv[h*64 + e], a slot already consumed
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = h * 64 + 2 * e;
          float d0, d1;
          f2_split(f2_add(f2_make(__uint_as_float(sv[col]), __uint_as_float(sv[col + 1])), neg_m), d0, d1);
          const float p0 = fast_exp2(d0), p1 = fast_exp2(d1);
          sv[h * 64 + e] = pack_bf16x2(p0, p1);
          lsum[e & 3] = f2_add(lsum[e & 3], f2_make(p0, p1));
        }
        tmem_st32p(tS + h * 32, sv + h * 64);
      }
      {
        float a0, a1;
        f2_split(f2_add(f2_add(lsum[0], lsum[1]), f2_add(lsum[2], lsum[3])), a0, a1);
        l_run += a0 + a1;
      }
      if (rescale) {
        // O has no MMA in flight here: PV_i(j-1) completed before S_i(j) was committed,
        // and PV_i(j) is issued only after this thread arrives on p_full below
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tO + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * corr);
          tmem_st32(tO + c * 32, v);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[i]);
    }
    // epilogue: O / l -> bf16 -> out
    if (alive && mbar_wait_warp(&o_full[i], 0, abort_flag)) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
      __nv_bfloat16* orow = nullptr;
      if (p.sv.G == 0) {
        orow = p.out + ((static_cast<int64_t>(state) * p.Nq + qr) * p.H + head) * D;
      } else if (qr < p.Nq) {
        // back to the rank whose sequence shard holds the row (the inverse all-to-all)
        int rk = 0;
        const int64_t off = shard_elem(p.sv, state, qr, head, D, rk);
        orow = p.o_sh[rk] + off;
      }
      uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + c * 32, v);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * inv, __uint_as_float(v[2 * e + 1]) * inv);
        if (qr < p.Nq) {
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

template <int D>
size_t smem_for(const AttnParams&) {
  using C = AttnCfg<D>;
  // at least half the SM's shared memory: one CTA per SM, so the 512-column
  // TMEM allocation never has to wait for a co-resident CTA
  return C::FIXED > 120 * 1024 ? C::FIXED : 120 * 1024;
}

template <int D>
int launch_t(const AttnParams& p, const CUtensorMap& q, const CUtensorMap* k, const CUtensorMap* v, int S,
             cudaStream_t s) {
  const size_t smem = smem_for<D>(p);
  auto kern = attn_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return static_cast<int>(e);
  dim3 grid((p.Nq + 255) / 256, p.nheads > 0 ? p.nheads : p.H, S);
  kern<<<grid, AttnCfg<D>::THREADS, smem, s>>>(q, k[0], v[0], k[1], v[1], k[2], v[2], k[3], v[3], p);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

size_t attend_smem_bytes(int D, const AttnParams& p) { return D == 128 ? smem_for<128>(p) : smem_for<64>(p); }

int launch_attend(int D, const AttnParams& p, const CUtensorMap& q, const CUtensorMap* k, const CUtensorMap* v,
                  int S, cudaStream_t s) {
  if (D == 128) return launch_t<128>(p, q, k, v, S, s);
  if (D == 64) return launch_t<64>(p, q, k, v, S, s);
  return static_cast<int>(cudaErrorInvalidValue);
}

}  // namespace ckv

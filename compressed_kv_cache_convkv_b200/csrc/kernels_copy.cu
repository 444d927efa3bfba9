// Streaming kernels: append of a block into the ring (bf16), permutation of the
// conv weights into the compression kernel's layout, and the mean-of-5
// compression variant.  All HBM-bound: 16-byte vector accesses, grids sized as
// a multiple of the SM count.
#include "convkv_internal.h"
#include "nvfp4.cuh"
#include "quant_div.cuh"
#include "rope.cuh"
#include "token_walk.h"

namespace ckv {

int token_grid_x(int T, int cols, int frames_yz) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int slabs = (cols + kTokenThreads - 1) / kTokenThreads;
  // about two waves of 8 resident CTAs per SM
  const int64_t ctas = static_cast<int64_t>(frames_yz) * slabs;
  int64_t walkers = (2LL * sms * 8 + ctas - 1) / ctas;
  if (walkers > T) walkers = T;
  if (walkers < 1) walkers = 1;
  return static_cast<int>(walkers * slabs);
}

namespace {

// Blocks along x for a launch whose y (and z) dimensions cover `frames` frames of
// `per_frame` work items: about 8 blocks per SM in total, at least one per frame.
int frame_grid_x(int64_t per_frame, int frames, int threads) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t need = (per_frame + threads - 1) / threads;
  int64_t want = (static_cast<int64_t>(sms) * 8 + frames - 1) / frames;
  if (want < 1) want = 1;
  return static_cast<int>(need < want ? need : want);
}

int grid_for(int64_t work_items, int threads) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t want = (work_items + threads - 1) / threads;
  int64_t cap = static_cast<int64_t>(sms) * 8;
  if (want < 1) want = 1;
  return static_cast<int>(want < cap ? want : cap);
}

// 16-byte vector e of frame f of state s in the block's [T][H][D] layout: in the plain
// tensor, or gathered from the sequence shard of the rank that holds the row (the
// all-to-all of k/v fused into the append; the shard may live in a peer's memory).
__device__ __forceinline__ const uint4* block_vec(const void* plain, const void* const* sh, const AppendParams& p,
                                                  int s, int f, int64_t e) {
  const int64_t fv = p.frame_elems / 8;
  if (p.sv.G == 0) return static_cast<const uint4*>(plain) + (static_cast<int64_t>(s) * p.b + f) * fv + e;
  const int vpr = p.H * p.D / 8;  // vectors per token
  const int64_t T = p.frame_elems / (static_cast<int64_t>(p.H) * p.D);
  const int64_t t = e / vpr;
  const int rem = static_cast<int>(e - t * vpr);
  const int h = rem / (p.D / 8);
  int r = 0;
  const int64_t off = shard_elem(p.sv, s, static_cast<int64_t>(f) * T + t, h, p.D, r);
  return static_cast<const uint4*>(sh[r]) + off / 8 + (rem - h * (p.D / 8));
}

// Append (SoulX-LiveAct blog, "ConvKV Memory": append-only KV -- only the new
// tokens' K/V are written, cached entries are never recomputed).
// k, v: [S][b*T][H][D] bf16 -> ring slot (slot0 + f) % R of each state.  K is also
// written rotated into ringKr at the same place: a window or current-block key
// keeps its RoPE position relative to every later query (both are stream
// positions), so it is rotated once here instead of at every attend.
// Table row pointers of token `tok` of a frame whose time index is table row t_row.
template <int D>
__device__ __forceinline__ dev::RopeRow rope_row_of(const float4* tables, int tab_t_rows, int tab_h_rows,
                                                    const FastDiv& div_gw, int grid_w, int t_row, int tok) {
  using RC = RopeCfg<D>;
  const float4* tab_h = tables + static_cast<int64_t>(tab_t_rows) * RC::UT;
  const float4* tab_w = tab_h + static_cast<int64_t>(tab_h_rows) * RC::UH;
  const int y = div_gw.div(tok);
  const int x = tok - y * grid_w;
  return dev::RopeRow{tables + static_cast<int64_t>(t_row) * RC::UT, tab_h + y * RC::UH, tab_w + x * RC::UW};
}

// grid = (x, states * b): y is the frame, x walks the 16-byte vectors of its heads
// [h0, h0 + nh).
template <int D>
__global__ void append_bf16_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                   uint4* __restrict__ ringK, uint4* __restrict__ ringV, AppendParams p) {
  constexpr int DV = D / 8;               // 16-byte vectors per head
  const int fv = static_cast<int>(p.frame_elems / 8);  // 16-byte vectors per frame
  const int nv = fv / p.H * p.nh;         // vectors of the appended heads per frame
  const int sf = blockIdx.y;              // state * b + frame
  const int s = sf / p.b;
  const int f = sf - s * p.b;
  int slot = p.slot0 + f;
  if (slot >= p.R) slot -= p.R;
  const int64_t dst0 = (static_cast<int64_t>(s) * p.R + slot) * fv;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += gridDim.x * blockDim.x) {
    const int ht = i / DV;                // token * nh + (head - h0)
    const int tok = p.div_nh.div(ht);
    const int e = (tok * p.H + p.h0 + (ht - tok * p.nh)) * DV + (i & (DV - 1));
    const uint4 kv = __ldcs(block_vec(k, p.k_sh, p, s, f, e));
    const uint4 vv = __ldcs(block_vec(v, p.v_sh, p, s, f, e));
    ringK[dst0 + e] = kv;
    ringV[dst0 + e] = vv;
    if (p.ringKr) {
      const dev::RopeRow rr =
          rope_row_of<D>(p.tables, p.tab_t_rows, p.tab_h_rows, p.div_grid_w, p.grid_w, p.t_row0 + f, tok);
      uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
      dev::rope_chunk<D, false>(w, e % DV, rr, 1.0f);
      static_cast<uint4*>(p.ringKr)[dst0 + e] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// Rotated copies of the reference frames and memory slots for the current time table
// (bit-identical to rotating them tile by tile in the attention: same table, same
// rounding).
// grid = (x, states * (r + m)): y is the frame; token walk (each thread owns one
// (head, 8-channel chunk) column, CTAs stride over the frame's tokens).
template <int D>
__global__ void rotate_keys_kernel(RotateParams p) {
  constexpr int DV = D / 8;
  constexpr int U = 2;                            // loads in flight per thread
  const int HDV = p.H * DV;
  const int T = static_cast<int>(p.frame_vecs / HDV);
  const int nf = p.r + p.m;
  const int fv = static_cast<int>(p.frame_vecs);
  const int s = blockIdx.y / nf;
  const int fi = blockIdx.y - s * nf;
  const uint4* src;
  uint4* dst;
  if (fi < p.r) {
    const int64_t off = (static_cast<int64_t>(s) * p.r + fi) * fv;
    src = static_cast<const uint4*>(p.sink_src) + off;
    dst = static_cast<uint4*>(p.sink_dst) + off;
  } else {
    int pos = p.pos0 + fi - p.r;
    if (pos >= p.C) pos -= p.C;
    const int64_t off = (static_cast<int64_t>(s) * p.C + pos) * fv;
    src = static_cast<const uint4*>(p.mem_src) + off;
    dst = static_cast<uint4*>(p.mem_dst) + off;
  }
  const int slabs = (HDV + blockDim.x - 1) / blockDim.x;
  const int walker = blockIdx.x / slabs, walkers = gridDim.x / slabs;
  const int hc = (blockIdx.x - walker * slabs) * blockDim.x + threadIdx.x;
  if (hc < HDV) {
    const int c = hc % DV;
    for (int tok0 = walker; tok0 < T; tok0 += U * walkers) {
      uint4 xs[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tok = tok0 + u * walkers;
        xs[u] = tok < T ? __ldg(src + tok * HDV + hc) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tok = tok0 + u * walkers;
        if (tok >= T) break;
        const dev::RopeRow rr =
            rope_row_of<D>(p.tables, p.tab_t_rows, p.tab_h_rows, p.div_grid_w, p.grid_w, fi, tok);
        uint32_t w[4] = {xs[u].x, xs[u].y, xs[u].z, xs[u].w};
        dev::rope_chunk<D, false>(w, c, rr, 1.0f);
        dst[tok * HDV + hc] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
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
// grid = (x, states, groups * 2 (K|V)).
__global__ void mean_bf16_kernel(const uint4* __restrict__ ringK, const uint4* __restrict__ ringV,
                                 uint4* __restrict__ memK, uint4* __restrict__ memV, ConvParams p,
                                 int64_t frame_vecs) {
  const int fv = static_cast<int>(frame_vecs);
  const int s = blockIdx.y;
  const int g = blockIdx.z >> 1, kv = blockIdx.z & 1;
  const uint4* src = kv ? ringV : ringK;
  uint4* dst = (kv ? memV : memK) + (static_cast<int64_t>(s) * p.C + p.grp[g].mem_pos) * fv;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < fv; e += gridDim.x * blockDim.x) {
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < kEvict; ++j) {
      const uint4 x = src[(static_cast<int64_t>(s) * p.R + p.grp[g].ring_slot[j]) * fv + e];
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
    dst[e] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ---------------------------------------------------------------------------
// Append in the fp8 format (model card, --fp8_kv_cache: the cache is stored in
// FP8 and dequantised to BF16 on use).  Per (state, K|V, frame, head):
//   scale = amax / 448 over the frame's [T, D] values (1 if amax == 0),
//   code  = e4m3(x / scale), IEEE fp32 divide, round-to-nearest-even, saturating.
// The block's bf16 values are also copied to staging: the current block is
// attended in bf16 and joins the window, e4m3, at the next append.

// pass 1: amax.  grid = (x, states * b, 2 (K|V)), token walk: each thread owns one
// (head, 8-channel chunk) column and keeps the running max of |x| over the tokens its
// CTA visits (a CTA's load step reads kTokenThreads * 16 contiguous bytes of a token);
// the D/8 lanes of a head then reduce by shuffles and one of them updates the frame's
// per-head maximum in global memory.
template <int D>
__global__ void append_amax_frames_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, AppendParams p) {
  constexpr int DV = D / 8;                       // lanes (vectors) per head
  constexpr int U = 4;                            // loads in flight per thread
  const int HDV = p.H * DV;                       // vectors per token
  const int NDV = p.nh * DV;                      // columns: the heads [h0, h0 + nh)
  const int T = static_cast<int>(p.frame_elems / HDV / 8);
  const int sf = blockIdx.y;
  const int s = sf / p.b;
  const int f = sf - s * p.b;
  const int kv = blockIdx.z;
  const int lane = threadIdx.x & 31;
  unsigned int* amax_f = p.amax + ((static_cast<int64_t>(s) * 2 + kv) * p.b + f) * p.H;
  const int slabs = (NDV + blockDim.x - 1) / blockDim.x;
  const int walker = blockIdx.x / slabs, walkers = gridDim.x / slabs;
  const int hc = (blockIdx.x - walker * slabs) * blockDim.x + threadIdx.x;
  const int col = p.h0 * DV + hc;                 // the column within the token
  uint32_t m = 0;
  if (hc < NDV) {
    for (int tok0 = walker; tok0 < T; tok0 += U * walkers) {
      uint4 x[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tok = tok0 + u * walkers;
        x[u] = tok < T ? __ldg(block_vec(kv ? v : k, kv ? p.v_sh : p.k_sh, p, s, f, static_cast<int64_t>(tok) * HDV + col))
                       : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t w[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          m = max(m, (w[q] & 0x7FFFu) << 16);   // |lo| as fp32 bits
          m = max(m, w[q] & 0x7FFF0000u);       // |hi| as fp32 bits
        }
      }
    }
  }
  // heads start at multiples of DV columns, slabs at multiples of 32, and DV divides 32
#pragma unroll
  for (int o = DV / 2; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (hc < NDV && (lane % DV) == 0 && m) atomicMax(&amax_f[col / DV], m);
}

// The block's K row chunk as written to staging: rotated at its stream position
// (frame f of the block at time-table row t_row0 + f) when the tables are given --
// the current block keeps its RoPE position relative to every later query, like
// the pre-rotated ring of the bf16 format -- else as is.  tok: the token within the
// frame; c: the 8-channel chunk within the head.
template <int D>
__device__ __forceinline__ uint4 staged_k(uint4 x, const AppendParams& p, int f, int tok, int c) {
  if (!p.tables) return x;
  const dev::RopeRow rr =
      rope_row_of<D>(p.tables, p.tab_t_rows, p.tab_h_rows, p.div_grid_w, p.grid_w, p.t_row0 + f, tok);
  uint32_t w[4] = {x.x, x.y, x.z, x.w};
  dev::rope_chunk<D, false>(w, c, rr, 1.0f);
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// pass 2: quantise into the ring, copy to staging (K rotated), record the scales.
// grid = (x, states * b, 2 (K|V)), token walk: each thread owns one (head h, chunk c)
// column, so the head's scale and its divisor are set up once per thread.
template <int D>
__global__ void append_quant_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, AppendParams p) {
  constexpr int DV = D / 8;
  constexpr int U = 2;                            // loads in flight per thread
  const int HDV = p.H * DV;                       // vectors per token
  const int NDV = p.nh * DV;                      // columns: the heads [h0, h0 + nh)
  const int T = static_cast<int>(p.frame_elems / HDV / 8);
  const int fv = static_cast<int>(p.frame_elems / 8);
  const int sf = blockIdx.y;
  const int s = sf / p.b;
  const int f = sf - s * p.b;
  const int kv = blockIdx.z;
  int slot = p.slot0 + f;
  if (slot >= p.R) slot -= p.R;
  const unsigned int* amax_f = p.amax + ((static_cast<int64_t>(s) * 2 + kv) * p.b + f) * p.H;
  uint4* stage = reinterpret_cast<uint4*>(p.stage[kv]) + (static_cast<int64_t>(s) * p.stage_frames + f) * fv;
  uint2* codes = reinterpret_cast<uint2*>(p.ring8[kv]) + (static_cast<int64_t>(s) * p.R + slot) * fv;
  const SharedDivisor d448 = make_divisor(448.0f);
  const int slabs = (NDV + blockDim.x - 1) / blockDim.x;
  const int walker = blockIdx.x / slabs, walkers = gridDim.x / slabs;
  const int hc = p.h0 * DV + (blockIdx.x - walker * slabs) * blockDim.x + threadIdx.x;
  if (hc < (p.h0 + p.nh) * DV) {
    const int h = hc / DV;
    const int c = hc - h * DV;
    const float amax = __uint_as_float(amax_f[h]);
    const float scale = amax > 0.0f ? div_rn(amax, d448) : 1.0f;
    const SharedDivisor ds = make_divisor(scale);
    if (walker == 0 && c == 0) p.ring_scale[((static_cast<int64_t>(s) * 2 + kv) * p.R + slot) * p.H + h] = scale;
    for (int tok0 = walker; tok0 < T; tok0 += U * walkers) {
      uint4 xs[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tok = tok0 + u * walkers;
        xs[u] = tok < T ? __ldg(block_vec(kv ? v : k, kv ? p.v_sh : p.k_sh, p, s, f, static_cast<int64_t>(tok) * HDV + hc))
                        : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tok = tok0 + u * walkers;
        if (tok >= T) break;
        const int e = tok * HDV + hc;
        const uint4 x = xs[u];
        stage[e] = kv == 0 ? staged_k<D>(x, p, f, tok, c) : x;
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t o[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint16_t lo, hi;
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
              : "=h"(lo)
              : "f"(div_rn(__uint_as_float(w[2 * q] & 0xFFFF0000u), ds)),
                "f"(div_rn(__uint_as_float(w[2 * q] << 16), ds)));
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
              : "=h"(hi)
              : "f"(div_rn(__uint_as_float(w[2 * q + 1] & 0xFFFF0000u), ds)),
                "f"(div_rn(__uint_as_float(w[2 * q + 1] << 16), ds)));
          o[q] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
        }
        codes[e] = make_uint2(o[0], o[1]);
      }
    }
  }
}

// NVFP4 pass 2: one thread per 16-channel block of a token's head: block scale,
// e2m1 codes into the ring, the bf16 values into staging (K rotated), the tensor
// scale once.
// grid = (x, states * b, 2 (K|V)); x walks the 16-channel blocks of the frame's heads
// [h0, h0 + nh).
template <int D>
__global__ void append_quant_fp4_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, AppendParams p) {
  constexpr int NB = D / fp4::kBlock;                      // blocks per token-head
  const int fv = static_cast<int>(p.frame_elems / 8);
  const int per_frame = static_cast<int>(p.frame_elems / fp4::kBlock / p.H * p.nh);
  const int sf = blockIdx.y;
  const int s = sf / p.b;
  const int f = sf - s * p.b;
  const int kv = blockIdx.z;
  int slot = p.slot0 + f;
  if (slot >= p.R) slot -= p.R;
  const int T = static_cast<int>(p.frame_elems / (static_cast<int64_t>(p.H) * D));
  const unsigned int* amax_f = p.amax + ((static_cast<int64_t>(s) * 2 + kv) * p.b + f) * p.H;
  uint4* stage = reinterpret_cast<uint4*>(p.stage[kv]) + (static_cast<int64_t>(s) * p.stage_frames + f) * fv;
  const int64_t row0 = (static_cast<int64_t>(s) * p.R + slot) * T * p.H;   // first token-head row of the slot
  for (int ib = blockIdx.x * blockDim.x + threadIdx.x; ib < per_frame; ib += gridDim.x * blockDim.x) {
    const int tl = ib / NB;                                    // token * nh + (h - h0)
    const int blk = ib - tl * NB;
    const int tok = p.div_nh.div(tl);
    const int h = p.h0 + (tl - tok * p.nh);
    const int th = tok * p.H + h;                              // token * H + h
    const int e0 = th * (D / 8) + blk * 2;                     // first 16-byte vector of the block
    const uint4 x0 = __ldg(block_vec(kv ? v : k, kv ? p.v_sh : p.k_sh, p, s, f, e0));
    const uint4 x1 = __ldg(block_vec(kv ? v : k, kv ? p.v_sh : p.k_sh, p, s, f, e0 + 1));
    stage[e0] = kv == 0 ? staged_k<D>(x0, p, f, tok, 2 * blk) : x0;
    stage[e0 + 1] = kv == 0 ? staged_k<D>(x1, p, f, tok, 2 * blk + 1) : x1;
    const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    float xs[fp4::kBlock];
    float a_b = 0.0f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      xs[2 * q] = __uint_as_float(w[q] << 16);
      xs[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
      a_b = fmaxf(a_b, fmaxf(fabsf(xs[2 * q]), fabsf(xs[2 * q + 1])));
    }
    const float g = fp4::tensor_scale(__uint_as_float(amax_f[h]));
    float e_b;
    const uint32_t sc = fp4::block_scale(a_b, g, fp4::block_divisor(g), e_b);
    const int64_t row = row0 + th;                              // token-head row in the ring
    reinterpret_cast<uint2*>(p.ring8[kv])[row * NB + blk] = fp4::encode_block(xs, e_b);
    p.ring_bs[kv][row * NB + blk] = static_cast<uint8_t>(sc);
    if (tok == 0 && blk == 0) p.ring_scale[((static_cast<int64_t>(s) * 2 + kv) * p.R + slot) * p.H + h] = g;
  }
}

}  // namespace

int launch_append_bf16(const AppendParams& p, const void* k, const void* v, void* ringK, void* ringV,
                       cudaStream_t s) {
  if (p.nh < 1 || p.h0 < 0 || p.h0 + p.nh > p.H) return static_cast<int>(cudaErrorInvalidValue);
  auto kern = p.D == 128 ? append_bf16_kernel<128> : append_bf16_kernel<64>;
  dim3 grid(frame_grid_x(p.frame_elems / 8 / p.H * p.nh, p.S * p.b, 256), p.S * p.b);
  kern<<<grid, 256, 0, s>>>(static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(ringK),
                            static_cast<uint4*>(ringV), p);
  return static_cast<int>(cudaGetLastError());
}

int launch_rotate_keys(int D, const RotateParams& p, cudaStream_t s) {
  const int frames = p.S * (p.r + p.m);
  if (frames == 0) return 0;
  auto kern = D == 128 ? rotate_keys_kernel<128> : rotate_keys_kernel<64>;
  const int T = static_cast<int>(p.frame_vecs / (static_cast<int64_t>(p.H) * (D / 8)));
  dim3 grid(token_grid_x(T, p.H * (D / 8), frames), frames);
  kern<<<grid, kTokenThreads, 0, s>>>(p);
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
  if (p.ngroups <= 0) return 0;
  dim3 grid(frame_grid_x(frame_vecs, p.S * 2 * p.ngroups, 256), p.S, 2 * p.ngroups);
  mean_bf16_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(ringK), static_cast<const uint4*>(ringV),
                                        static_cast<uint4*>(p.memK), static_cast<uint4*>(p.memV), p, frame_vecs);
  return static_cast<int>(cudaGetLastError());
}

int launch_append_fp8(const AppendParams& p, const void* k, const void* v, cudaStream_t s) {
  if (p.nh < 1 || p.h0 < 0 || p.h0 + p.nh > p.H) return static_cast<int>(cudaErrorInvalidValue);
  cudaError_t e = cudaMemsetAsync(p.amax, 0, sizeof(unsigned int) * p.S * 2 * p.b * p.H, s);
  if (e != cudaSuccess) return static_cast<int>(e);
  {
    auto kern = p.D == 128 ? append_amax_frames_kernel<128> : append_amax_frames_kernel<64>;
    const int T = static_cast<int>(p.frame_elems / (static_cast<int64_t>(p.H) * p.D));
    dim3 g1(token_grid_x(T, p.nh * (p.D / 8), 2 * p.S * p.b), p.S * p.b, 2);
    kern<<<g1, kTokenThreads, 0, s>>>(static_cast<const uint4*>(k), static_cast<const uint4*>(v), p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return static_cast<int>(e);
  if (p.fp4) {
    auto kern = p.D == 128 ? append_quant_fp4_kernel<128> : append_quant_fp4_kernel<64>;
    dim3 grid(frame_grid_x(p.frame_elems / fp4::kBlock / p.H * p.nh, 2 * p.S * p.b, 256), p.S * p.b, 2);
    kern<<<grid, 256, 0, s>>>(static_cast<const uint4*>(k), static_cast<const uint4*>(v), p);
    return static_cast<int>(cudaGetLastError());
  }
  auto kern = p.D == 128 ? append_quant_kernel<128> : append_quant_kernel<64>;
  const int T = static_cast<int>(p.frame_elems / (static_cast<int64_t>(p.H) * p.D));
  dim3 grid(token_grid_x(T, p.nh * (p.D / 8), 2 * p.S * p.b), p.S * p.b, 2);
  kern<<<grid, kTokenThreads, 0, s>>>(static_cast<const uint4*>(k), static_cast<const uint4*>(v), p);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace ckv

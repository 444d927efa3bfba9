// Dequantisation to BF16 on use (model card, Command Line Arguments, --fp8_kv_cache:
// the KV cache is stored in FP8 and dequantised to BF16 when it is used).  Once per
// attend and group of states, the e4m3 / NVFP4 codes of the window frames and memory
// slots are turned into a bf16 scratch -- K rotated for its reset RoPE position --
// which the attention then reads like the bf16 cache.  Each tile is thus converted
// once, not once per query block that reads it.
//
// Every value is bf16(fp32(code * scale)): e4m3 codes with the per-(frame or slot,
// head) scale, NVFP4 codes with fp32(s_b * g).  K is then rotated like every other
// key (rope.cuh) with time-table row r + i for the i-th frame of [memory | window].
#include "convkv_internal.h"
#include "lowp_codes.cuh"
#include "nvfp4.cuh"
#include "rope.cuh"
#include "token_walk.h"

namespace ckv {
namespace {

// grid = (x, states * (m + w), 2 (K|V)), token walk: each thread owns one (head h,
// 8-channel chunk c) column (its scale and conversion path are fixed for the whole
// walk), CTAs stride over the frame's tokens.
template <int D>
__global__ void dequant_kernel(DequantParams p) {
  using RC = RopeCfg<D>;
  constexpr int DV = D / 8;                      // 16-byte bf16 vectors per head
  constexpr int U = 4;                           // code loads in flight per thread
  const int HDV = p.H * DV;
  const int T = static_cast<int>(p.frame_elems / HDV / 8);
  const int nf = p.m + p.w;
  const int fv = static_cast<int>(p.frame_elems / 8);
  const int sl = blockIdx.y / nf;                // state within the group
  const int fi = blockIdx.y - sl * nf;           // frame in attend order
  const int state = p.state0 + sl;
  const int kv = blockIdx.z;
  const bool mem = fi < p.m;
  int slot = mem ? p.pos0 + fi : p.ring0 + fi - p.m;
  const int nsl = mem ? p.C : p.R;
  if (slot >= nsl) slot -= nsl;
  const int64_t frame = static_cast<int64_t>(state) * nsl + slot;
  const float* scl = (mem ? p.mem_scale : p.ring_scale) + ((static_cast<int64_t>(state) * 2 + kv) * nsl + slot) * p.H;
  const uint8_t* codes = mem ? p.mem8[kv] : p.ring8[kv];
  const uint2* codes8 = reinterpret_cast<const uint2*>(codes + frame * p.frame_elems);
  const uint32_t* codes4 = reinterpret_cast<const uint32_t*>(codes + frame * (p.frame_elems / 2));
  const uint8_t* bsf = (mem ? p.mem_bs[kv] : p.ring_bs[kv]) + frame * (p.frame_elems / 16);
  uint4* out = static_cast<uint4*>(p.out[kv]) + (static_cast<int64_t>(sl) * p.out_frames + fi) * fv;
  const float4* tab_h = p.tables + static_cast<int64_t>(p.tab_t_rows) * RC::UT;
  const float4* tab_w = tab_h + static_cast<int64_t>(p.tab_h_rows) * RC::UH;
  const float4* tab_t = p.tables + static_cast<int64_t>(p.r + fi) * RC::UT;
  const int slabs = (HDV + blockDim.x - 1) / blockDim.x;
  const int walker = blockIdx.x / slabs, walkers = gridDim.x / slabs;
  const int hc = (blockIdx.x - walker * slabs) * blockDim.x + threadIdx.x;
  if (hc < HDV) {
    const int h = hc / DV;
    const int c = hc - h * DV;                   // 8-channel chunk within the head
    const float sc = __ldg(scl + h);
    const bool fold8 = sc < dev::kE4m3FoldLimit;
    const float sc8 = fold8 ? sc * dev::kTwo120 : sc;
    for (int tok0 = walker; tok0 < T; tok0 += U * walkers) {
      uint2 cw[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tok = tok0 + u * walkers;
        const int e = tok * HDV + hc;
        if (tok >= T) {
          cw[u] = make_uint2(0, 0);
        } else if (p.fp4) {
          cw[u] = make_uint2(__ldg(codes4 + e), __ldg(bsf + static_cast<int64_t>(tok * p.H + h) * (D / 16) + (c >> 1)));
        } else {
          cw[u] = __ldg(codes8 + e);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tok = tok0 + u * walkers;
        if (tok >= T) break;
        uint32_t o[4];
        if (p.fp4) {
          const float e_b = __fmul_rn(fp4::e4m3_to_f32(cw[u].y), sc);
          if (e_b < dev::kFp4FoldLimit) {
            dev::e2m1x8_to_bf16<true>(cw[u].x, e_b * dev::kTwo112, o);
          } else {
            dev::e2m1x8_to_bf16<false>(cw[u].x, e_b, o);
          }
        } else if (fold8) {
          dev::e4m3x8_to_bf16<true>(cw[u].x, cw[u].y, sc8, o);
        } else {
          dev::e4m3x8_to_bf16<false>(cw[u].x, cw[u].y, sc8, o);
        }
        if (kv == 0) {
          const int y = p.div_grid_w.div(tok);
          const int x = tok - y * p.grid_w;
          const dev::RopeRow rr{tab_t, tab_h + y * RC::UH, tab_w + x * RC::UW};
          dev::rope_chunk<D, false>(o, c, rr, 1.0f);
        }
        out[tok * HDV + hc] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

}  // namespace

int launch_dequant(int D, const DequantParams& p, int states, cudaStream_t s) {
  const int frames = states * (p.m + p.w);
  if (frames == 0) return 0;
  if (frames > 65535) return static_cast<int>(cudaErrorInvalidValue);
  const int T = static_cast<int>(p.frame_elems / (static_cast<int64_t>(p.H) * D));
  dim3 grid(token_grid_x(T, p.H * (D / 8), 2 * frames), frames, 2);
  if (D == 128) {
    dequant_kernel<128><<<grid, kTokenThreads, 0, s>>>(p);
  } else if (D == 64) {
    dequant_kernel<64><<<grid, kTokenThreads, 0, s>>>(p);
  } else {
    return static_cast<int>(cudaErrorInvalidValue);
  }
  return static_cast<int>(cudaGetLastError());
}

}  // namespace ckv

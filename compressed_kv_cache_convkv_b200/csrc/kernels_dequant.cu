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

namespace ckv {
namespace {

// grid = (x over the frame's 16-byte output vectors, states * (m + w), 2 (K|V))
template <int D>
__global__ void dequant_kernel(DequantParams p) {
  using RC = RopeCfg<D>;
  constexpr int DV = D / 8;                      // 16-byte bf16 vectors per head
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
  const uint8_t* bsb = mem ? p.mem_bs[kv] : p.ring_bs[kv];
  uint4* out = static_cast<uint4*>(p.out[kv]) + (static_cast<int64_t>(sl) * p.out_frames + fi) * fv;
  const float4* tab_h = p.tables + static_cast<int64_t>(p.tab_t_rows) * RC::UT;
  const float4* tab_w = tab_h + static_cast<int64_t>(p.tab_h_rows) * RC::UH;
  constexpr int U = 4;                            // code loads in flight per thread
  const int stride = gridDim.x * blockDim.x;
  for (int e0 = blockIdx.x * blockDim.x + threadIdx.x; e0 < fv; e0 += U * stride) {
    uint2 cw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int e = e0 + u * stride;
      if (e >= fv) {
        cw[u] = make_uint2(0, 0);
      } else if (p.fp4) {
        cw[u].x = __ldg(reinterpret_cast<const uint32_t*>(codes + frame * (p.frame_elems / 2)) + e);
        cw[u].y = 0;
      } else {
        cw[u] = __ldg(reinterpret_cast<const uint2*>(codes + frame * p.frame_elems) + e);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int e = e0 + u * stride;
      if (e >= fv) break;
      const int hv = e / DV;                        // token * H + head
      const int c = e - hv * DV;                    // 8-channel chunk within the head
      const int tok = p.div_heads.div(hv);
      const int h = hv - tok * p.H;
      const float sc = __ldg(scl + h);
      uint32_t o[4];
      if (p.fp4) {
        const uint32_t word = cw[u].x;
        const uint8_t sb = __ldg(bsb + frame * (p.frame_elems / 16) + static_cast<int64_t>(hv) * (D / 16) + (c >> 1));
        const float e_b = __fmul_rn(fp4::e4m3_to_f32(sb), sc);
        if (e_b < dev::kFp4FoldLimit) {
          dev::e2m1x8_to_bf16<true>(word, e_b * dev::kTwo112, o);
        } else {
          dev::e2m1x8_to_bf16<false>(word, e_b, o);
        }
      } else {
        const uint2 w = cw[u];
        if (sc < dev::kE4m3FoldLimit) {
          dev::e4m3x8_to_bf16<true>(w.x, w.y, sc * dev::kTwo120, o);
        } else {
          dev::e4m3x8_to_bf16<false>(w.x, w.y, sc, o);
        }
      }
      if (kv == 0) {
        const int y = p.div_grid_w.div(tok);
        const int x = tok - y * p.grid_w;
        const dev::RopeRow rr{p.tables + static_cast<int64_t>(p.r + fi) * RC::UT, tab_h + y * RC::UH,
                              tab_w + x * RC::UW};
        dev::rope_chunk<D, false>(o, c, rr, 1.0f);
      }
      out[e] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace

int launch_dequant(int D, const DequantParams& p, int states, cudaStream_t s) {
  const int frames = states * (p.m + p.w);
  if (frames == 0) return 0;
  if (frames > 65535) return static_cast<int>(cudaErrorInvalidValue);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t need = (p.frame_elems / 8 + 255) / 256;
  int64_t want = (static_cast<int64_t>(sms) * 8 + 2 * frames - 1) / (2 * frames);
  if (want < 1) want = 1;
  dim3 grid(static_cast<unsigned>(need < want ? need : want), frames, 2);
  if (D == 128) {
    dequant_kernel<128><<<grid, 256, 0, s>>>(p);
  } else if (D == 64) {
    dequant_kernel<64><<<grid, 256, 0, s>>>(p);
  } else {
    return static_cast<int>(cudaErrorInvalidValue);
  }
  return static_cast<int>(cudaGetLastError());
}

}  // namespace ckv

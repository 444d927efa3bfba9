// Internal interface between the host library (convkv_host.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace ckv {

constexpr int kEvict = 5;       // eviction group = conv kernel = conv stride (5:1)
constexpr int kMaxSegs = 6;     // key segments of one attend (reference 1 + memory 2 + ring 2 + staging 1)
constexpr int kMaxGroups = 16;  // eviction groups one append may compress

// RoPE channel pairs per axis for head_dim D: row and column floor(D/6), time the rest
__host__ __device__ constexpr int rope_pairs_h(int D) { return D / 6; }
__host__ __device__ constexpr int rope_pairs_t(int D) { return (D - 4 * (D / 6)) / 2; }
// 16-byte table units of an axis whose pairs are global pairs [g, g + n)
__host__ __device__ constexpr int rope_units(int g, int n) { return (g + n + 1) / 2 - g / 2; }

// Division of a non-negative int (< 2^31) by a fixed divisor d (1 <= d < 2^31) with a
// multiply-high, shift and add (Granlund and Montgomery, "Division by invariant
// integers using multiplication", PLDI 1994): l = ceil(log2 d),
// m = floor(2^32 (2^l - d) / d) + 1, n / d = (mulhi(m, n) + n) >> l.
struct FastDiv {
  uint32_t d = 1, m = 1, l = 0;
  FastDiv() = default;
  __host__ explicit FastDiv(uint32_t div) : d(div) {
    while ((1u << l) < d) ++l;
    m = static_cast<uint32_t>((((uint64_t(1) << 32) * ((uint64_t(1) << l) - d)) / d) + 1);
  }
  __device__ __forceinline__ int div(int n) const {
    const uint32_t t = __umulhi(m, static_cast<uint32_t>(n));
    return static_cast<int>((t + static_cast<uint32_t>(n)) >> l);
  }
};

// Device status word values (written by kernels, read by convkv_status()).
constexpr int kStatusOk = 0;
constexpr int kStatusTimeout = 1;

// One contiguous run of key rows in one buffer (all bf16, K stored rotated).
struct KeySeg {
  int buf;     // tensor map pair: 0 ring (bf16 format) or dequantised scratch (e4m3 / NVFP4),
               // 1 memory, 2 current-block staging (e4m3 / NVFP4), 3 reference frames
  int row0;    // first row (token) in that buffer, a frame boundary
  int nrows;   // rows = frames * T
  int local;   // 1 if the buffer holds only the launch's group of states (the scratch)
};

// A block's rows (frames * T tokens) split into G contiguous sequence shards, one
// per rank, each holding every head of its rows: shard r is [S][off[r+1]-off[r]][Ht][D]
// bf16 and this handle owns heads [h0, h0 + H) of Ht.  G == 0: not sharded, the
// block is one [S][rows][H][D] tensor.
constexpr int kMaxRanks = 8;
struct ShardView {
  int G, Ht, h0;
  int64_t off[kMaxRanks + 1];
};

// Element offset (in bf16 units) of (state s, block row `row`, local head h, channel 0)
// inside shard `r`, the shard that holds the row.
__host__ __device__ __forceinline__ int64_t shard_elem(const ShardView& v, int s, int64_t row, int h, int D,
                                                       int& r) {
  r = 0;
#pragma unroll
  for (int q = 1; q < kMaxRanks; ++q)
    if (q < v.G && row >= v.off[q]) r = q;
  const int64_t n = v.off[r + 1] - v.off[r];
  return ((static_cast<int64_t>(s) * n + (row - v.off[r])) * v.Ht + v.h0 + h) * D;
}

struct AttnParams {
  int H, T, grid_w, Nq;   // Nq = query rows per state (frames * T)
  int tq0;                // RoPE time index of the current block's first frame (m + w)
  int nseg, ntiles;
  KeySeg seg[kMaxSegs];
  int tab_t_rows, tab_h_rows, tab_w_rows;  // rows (positions) of the three RoPE tables
  // RoPE tables, one per axis, rows of 16-byte units: unit u of a row holds
  // (cos, cos, sin, sin) of the two channel pairs 2k, 2k+1 (k = floor(g/2) + u, g =
  // the axis' first global pair) that belong to the axis, zeros for a pair that
  // does not; [t rows][units_t] ++ [grid_h][units_h] ++ [grid_w][units_w]
  const float4* tables;
  __nv_bfloat16* out;     // [S][Nq][H][D]
  float q_scale;          // log2(e) / sqrt(D), folded into the rotated queries
  int state0;             // first state of the launch's group (grid z walks the group)
  int head0, nheads;      // heads [head0, head0 + nheads) (grid y); nheads 0: all H
  int* status;
  // sequence-sharded queries and outputs (sv.G > 0): rows of the block are read from
  // and written to the G ranks' shards (peer memory on a multi-GPU node)
  ShardView sv;
  const __nv_bfloat16* q_sh[kMaxRanks];
  __nv_bfloat16* o_sh[kMaxRanks];
};

struct ConvGroup {
  int ring_slot[kEvict];  // physical ring slots of the 5 frames, oldest first
  int mem_pos;            // destination memory position
};

struct ConvParams {
  int H, T, S, C, R, ngroups;
  ConvGroup grp[kMaxGroups];
  void* memK;             // bf16 [S][C*T][H][D], or e4m3 in the fp8 format
  void* memV;
  int* status;
  // fp8 format: e4m3 ring input with per-(frame, head) scales; the conv pass keeps its
  // fp32 outputs and their per-(slot, head) amax, a second kernel quantises them
  float* acc;                 // fp32 conv outputs [S][ngroups][2][T][H][D] of this launch
  const uint8_t* ring8[2];    // e4m3 K, V rings [S][R*T][H][D]
  const float* ring_scale;    // [S][2][R][H]
  unsigned int* amax;         // [S][2][ngroups][H] fp32 bit patterns (scratch, zeroed before pass 1)
  float* mem_scale;           // [S][2][C][H]
  // NVFP4 format: ring8 / memK / memV hold e2m1 code pairs [..][D/2], scales as below
  const uint8_t* ring_bs[2];  // e4m3 block scales of the ring [S][R*T][H][D/16]
  uint8_t* mem_bs[2];         // e4m3 block scales of the memory [S][C*T][H][D/16]
};

struct AppendParams {
  int S, b, R, slot0;         // states, frames, ring frames, ring slot of frame 0
  int64_t frame_elems;        // T * H * D
  // heads [h0, h0 + nh) of each token are appended (nh >= 1); div_nh divides by nh
  int h0, nh;
  FastDiv div_nh;
  // fp8 format
  int H, D;
  unsigned int* amax;         // [S][2][b][H] fp32 bit patterns (scratch, zeroed before the amax pass)
  uint8_t* ring8[2];          // e4m3 K, V rings
  float* ring_scale;          // [S][2][R][H]
  uint8_t* ring_bs[2];        // NVFP4: e4m3 block scales [S][R*T][H][D/16] (ring8 then holds e2m1 pairs)
  int fp4;                    // 1: NVFP4 format
  void* stage[2];             // bf16 K, V current-block staging [S][stage_frames*T][H][D]
  int stage_frames;           // frames per state in the staging buffers (max block)
  // sequence-sharded K, V (sv.G > 0): the block's rows are gathered from the G ranks'
  // shards (peer memory on a multi-GPU node) instead of the k, v tensors
  ShardView sv;
  const void* k_sh[kMaxRanks];
  const void* v_sh[kMaxRanks];
  // bf16 format: K is also stored rotated (ringKr) with the RoPE tables of the step;
  // frame f of the block sits at table row t_row0 + f, token s at (s / grid_w, s % grid_w)
  void* ringKr;
  const float4* tables;
  int tab_t_rows, tab_h_rows, t_row0, grid_w;
  FastDiv div_heads, div_grid_w;   // by H and by grid_w (token -> head, row, column)
};

// Rotation of the cached keys that are not stored rotated at append: the r reference
// frames and the m stored memory slots, whose RoPE positions move with every eviction
// (RoPE Reset).  Frame i < r is reference frame i (table row i); frame i >= r is the
// memory position (pos0 + i - r) mod C (table row i).  src/dst: [S][frames*T][H][D] bf16.
struct RotateParams {
  int S, r, m, C, pos0;
  int64_t frame_vecs;          // 16-byte vectors per frame (T * H * D / 8)
  int H, grid_w;
  const void* sink_src;
  void* sink_dst;
  const void* mem_src;
  void* mem_dst;
  const float4* tables;
  int tab_t_rows, tab_h_rows;
  FastDiv div_heads, div_grid_w;
};

// Dequantisation of the e4m3 / NVFP4 window and memory into a bf16 scratch, once per
// attend and group of states: frame i < m is the memory position (pos0 + i) mod C,
// frame i >= m the ring slot (ring0 + i - m) mod R; every value is bf16(fp32(code *
// scale)) (NVFP4 scale fp32(s_b * g)), K rotated with time-table row r + i.  Output
// [S_group][out_frames * T][H][D] bf16 for K and V, frames in attend order.
struct DequantParams {
  int state0, m, w, r, C, R, H, grid_w, pos0, ring0, out_frames, fp4;
  int64_t frame_elems;            // T * H * D
  const uint8_t* ring8[2];        // codes: e4m3 [S][R*T][H][D], or NVFP4 pairs [..][D/2]
  const uint8_t* mem8[2];
  const float* ring_scale;        // [S][2][R][H]
  const float* mem_scale;         // [S][2][C][H]
  const uint8_t* ring_bs[2];      // NVFP4 e4m3 block scales [..][D/16]
  const uint8_t* mem_bs[2];
  void* out[2];
  const float4* tables;
  int tab_t_rows, tab_h_rows;
  FastDiv div_heads, div_grid_w;
};

// Kernel launchers (return cudaError_t of the launch).
int launch_dequant(int D, const DequantParams& p, int states, cudaStream_t s);
int launch_rotate_keys(int D, const RotateParams& p, cudaStream_t s);
int launch_append_bf16(const AppendParams& p, const void* k, const void* v, void* ringK, void* ringV,
                       cudaStream_t s);
int launch_permute_weights(const void* src, void* dst, int S, int H, int D, cudaStream_t s);
int launch_conv_bf16(int D, const ConvParams& p, const CUtensorMap& ringK, const CUtensorMap& ringV,
                     const CUtensorMap& wmap, cudaStream_t s);
int launch_mean_bf16(int D, const ConvParams& p, const void* ringK, const void* ringV, cudaStream_t s);
// codesK, codesV: TMA maps of the ring's code tiles (one head's 128 rows of codes)
int launch_conv_fp8(int D, const ConvParams& p, const CUtensorMap& codesK, const CUtensorMap& codesV,
                    const CUtensorMap& wmap, cudaStream_t s);
int launch_conv_fp4(int D, const ConvParams& p, const CUtensorMap& codesK, const CUtensorMap& codesV,
                    const CUtensorMap& wmap, cudaStream_t s);
int launch_append_fp8(const AppendParams& p, const void* k, const void* v, cudaStream_t s);
// k, v: tensor maps of buffers 0..3 (ring or scratch, memory, staging, reference frames);
// S: states in the launch (from p.state0)
int launch_attend(int D, const AttnParams& p, const CUtensorMap& q, const CUtensorMap* k,
                  const CUtensorMap* v, int S, cudaStream_t s);
size_t attend_smem_bytes(int D, const AttnParams& p);
size_t conv_smem_bytes(int D);

}  // namespace ckv

// Host side of the ConvKV C ABI: configuration checks, the integer bookkeeping
// of the ring window / FIFO memory (bit-exact, independent of stream length),
// the single device arena, RoPE tables, TMA descriptors and launch order.
//
// Bookkeeping (SoulX-LiveAct blog walk-through, sections "ConvKV Memory" and
// "Streaming Pipeline"; aiboss88.com summary, ConvKV bullet, for the 5:1 ratio):
//   P  frames promoted into the window so far, E frames evicted, S slots made.
//   append(b): P += b_prev; while P - E > W: compress frames [E, E+5) into slot
//              S (memory position S mod C), E += 5, S += 1; the new block goes to
//              ring slots (P + f) mod R with R = W + max(b1, b).
//   attend:    keys = the r reference frames at time 0..r-1 (r = sink_frames, given
//              once, never evicted), stored slots S-m .. S-1 (m = min(S, C)) at
//              time r..r+m-1, then frames E .. P+b-1 at time r + m + (f - E).
//
// RoPE is relative, so the time table of a step may hold any common shift of these
// indices.  Each append rebuilds it for absolute positions B0 + i, B0 = E - r - m
// (+ t_offset): table row i then serves reset time index i, and a window or
// current frame's row is its stream index q - B0, so a key rotated at append time
// at stream position q stays valid at every later attend (bf16 format: the ring
// keeps an un-rotated K for the conv and a rotated copy for the attention).
#include <cmath>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/convkv.h"
#include "convkv_internal.h"

using namespace ckv;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// A unit of the host-buffer pipeline: states [g0, g0 + n) with heads [h0, h0 + nh);
// a head range narrower than H only ever covers one state.
struct IoChunk {
  int g0, n, h0, nh;
};

}  // namespace

struct convkv {
  convkv_cfg cfg{};
  int H = 0, D = 0, T = 0, gh = 0, gw = 0, b1 = 0, bn = 0, Bmax = 0, W = 0, C = 0, R = 0, S = 0, Rs = 0;
  int G = 1, g = 0;  // sequence-parallel group size and this handle's rank
  int PT = 0, PH = 0, PW = 0, tab_t_rows = 0;
  // fp8: the ring and memory are stored in a low-precision format (e4m3, or NVFP4 when fp4)
  bool dry = false, mean = false, fp8 = false, fp4 = false, host_io = false, sink_set = false, prerot = false;
  // bookkeeping
  int64_t P = 0, E = 0, Sn = 0, blocks = 0;
  int bcur = 0, last_groups = 0;
  // device memory
  void* arena = nullptr;
  size_t arena_bytes = 0;
  void *ringK = nullptr, *ringV = nullptr, *memK = nullptr, *memV = nullptr, *weights = nullptr;
  void* ringKr = nullptr;           // bf16 format: K of the ring rotated at its stream position
  // rotated copies of the keys whose RoPE positions move with every eviction: the
  // memory slots (bf16 format) and the reference frames (both formats), refreshed by
  // the append whenever the time table's base moves
  void *memKr = nullptr, *sinkKr = nullptr;
  int64_t rot_B0 = INT64_MIN;       // table base the rotated copies were made with
  bool rot_sink_stale = false;      // reference frames given since the last rotation
  std::vector<float4> tab_t_host;   // time table rows of the current step (host copy)
  // fp8 format: ringK/ringV/memK/memV hold e4m3 codes; scales per (state, K|V, slot, head)
  float *ring_scale = nullptr, *mem_scale = nullptr;
  void *stageK = nullptr, *stageV = nullptr;  // bf16 copy of the current block
  // NVFP4: ringK/ringV/memK/memV hold e2m1 pairs; e4m3 block scales per 16 channels
  uint8_t *ringBK = nullptr, *ringBV = nullptr, *memBK = nullptr, *memBV = nullptr;
  void *sinkK = nullptr, *sinkV = nullptr;    // bf16 reference frames, both formats
  void *scrK = nullptr, *scrV = nullptr;      // e4m3 / NVFP4: bf16 scratch [Sg][(C + W) * T][H][D]
  int Sg = 0;                                 // states per dequantise-and-attend group
  int sms = 148;                              // SMs of the device (148 for a dry-run handle)
  unsigned int* amax = nullptr;               // amax scratch of the quantisation passes
  float* convacc = nullptr;                   // e4m3 / NVFP4: fp32 conv outputs of one append
  int gmax = 0;                               // eviction groups one append can produce
  float4* tables = nullptr;
  int* status = nullptr;
  void *io_q = nullptr, *io_k = nullptr, *io_v = nullptr, *io_out = nullptr;
  // host I/O (CONVKV_FLAG_HOST_IO): the *_host entry points copy by chunks (of states,
  // or of one state's heads) on their own streams, and each chunk's kernels wait only
  // for that chunk's copy, so copies in both directions overlap the kernels of other
  // chunks -- and of the previous call's chunks: a chunk's staging is refilled as soon
  // as the previous call's kernels and copy back of that chunk are done
  cudaStream_t io_in = nullptr, io_back = nullptr;
  // n = io_nmax events each: [c] chunk c copied in (io_in), [n + c] chunk c's kernels
  // done (stream), [2n + c] chunk c's outputs copied back (io_back)
  std::vector<cudaEvent_t> io_ev;
  int io_nmax = 0;
  // chunk plans: [0] for a call that follows a synchronised one (ramps up from one
  // state), [1] for a queued step that follows a queued step (steady chunks)
  std::vector<IoChunk> io_plan[2];
  std::vector<IoChunk> io_chunks;  // the current call's plan, in stream order
  int io_nchunks = 0;
  std::vector<IoChunk> io_last;    // the previous host-buffer call's plan
  int io_frames = 0;               // ... and its block frames
  bool io_inflight = false;        // a queued step may still run
  bool io_pending = false;         // the next ring append reads io_k / io_v chunk by chunk
  bool io_defer = false;           // the ring append is left to the caller (convkv_step_host)
  AppendParams io_ap{};            // ... with these parameters
  CUtensorMap mapRingK{}, mapRingV{}, mapRingKr{}, mapMemK{}, mapMemV{}, mapW{}, mapStageK{}, mapStageV{}, mapSinkK{},
      mapSinkV{};
  // e4m3 / NVFP4: code tiles of the ring (read by the conv), and the bf16 scratch the
  // window and memory are dequantised into for each group of Sg states
  CUtensorMap mapRingCK{}, mapRingCV{}, mapScrK{}, mapScrV{};
  CUtensorMap mapMemKr{}, mapSinkKr{};
  cudaStream_t stream = nullptr;
  int64_t launches = 0;
  int last_cuda = 0;
  // host-side failure injection (tests): the fail_at-th launch step of the next
  // append reports a launch failure instead of running
  int fail_at = -1, steps = 0;
  // set when an append failed after rolling back its counters: a conv of that call
  // may already have rewritten a memory position, so attends wait for the next
  // successful append
  bool need_append = false;

  int cuda_fail(cudaError_t e) {
    last_cuda = static_cast<int>(e);
    return CONVKV_ERR_CUDA;
  }
  // Called before every launch step of an append (also in dry-run mode, where the
  // step itself is skipped); returns the injected error once when armed.
  cudaError_t step_gate() {
    if (fail_at >= 0 && steps++ == fail_at) {
      fail_at = -1;
      return cudaErrorLaunchFailure;
    }
    return cudaSuccess;
  }
  int64_t frame_elems() const { return static_cast<int64_t>(T) * H * D; }
  // attention CTAs per head and state of a steady block (one per 256 query rows)
  int64_t ctas_per_head() const { return (static_cast<int64_t>(bn) * T + 255) / 256; }
  cudaEvent_t ev_in(int c) const { return io_ev[c]; }
  cudaEvent_t ev_done(int c) const { return io_ev[io_nmax + c]; }
  cudaEvent_t ev_out(int c) const { return io_ev[2 * io_nmax + c]; }
  // The previous host-buffer call's chunk whose events cover the staging region of the
  // current call's chunk c for blocks of `frames` frames: the chunk that holds the
  // region's last (state, head) -- the streams run a call's chunks in order, so its
  // events also cover every earlier chunk -- or, when the block size (the staging
  // layout) changed, the previous call's last chunk.
  int io_prev(int c, int frames) const {
    const int n = static_cast<int>(io_last.size());
    if (n == 0) return 0;
    if (frames != io_frames) return n - 1;
    const IoChunk& k = io_chunks[c];
    const int s = k.g0 + k.n - 1, hd = k.h0 + k.nh - 1;
    for (int p = 0; p < n; ++p) {
      const IoChunk& q = io_last[p];
      if (s >= q.g0 && s < q.g0 + q.n && hd >= q.h0 && hd < q.h0 + q.nh) return p;
    }
    return n - 1;
  }
  // Start a host-buffer call: a queued step that follows a queued step takes the steady plan.
  void io_begin(bool queued) {
    io_chunks = io_plan[queued && io_inflight ? 1 : 0];
    io_nchunks = static_cast<int>(io_chunks.size());
  }
  void io_end(int frames, bool queued) {
    io_last = io_chunks;
    io_frames = frames;
    io_inflight = queued;
  }
  int m() const { return static_cast<int>(Sn < C ? Sn : C); }
  int w() const { return static_cast<int>(P - E); }
};

namespace {

int encode_4d(CUtensorMap* map, void* ptr, int D, int H, int64_t rows, int S) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return CONVKV_ERR_CUDA;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(S)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2,
                           static_cast<cuuint64_t>(rows) * H * D * 2};
  cuuint32_t box[4] = {64, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, ptr, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CONVKV_OK : CONVKV_ERR_CUDA;
}

// Codes of the e4m3 / NVFP4 cache [S][rows][H][cb] bytes: one box is 128 rows of one
// head's cb code bytes, written with the cb-byte swizzle (cb = 128, 64 or 32).
int encode_codes(CUtensorMap* map, void* ptr, int cb, int H, int64_t rows, int S) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return CONVKV_ERR_CUDA;
  const CUtensorMapSwizzle sw = cb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                          : (cb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  if (cb != 128 && cb != 64 && cb != 32) return CONVKV_ERR_UNSUPPORTED;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(cb), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(S)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(cb), static_cast<cuuint64_t>(H) * cb,
                           static_cast<cuuint64_t>(rows) * H * cb};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(cb), 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CONVKV_OK : CONVKV_ERR_CUDA;
}

int encode_weights(CUtensorMap* map, void* ptr, int D, int H, int S) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return CONVKV_ERR_CUDA;
  const cuuint64_t rows = static_cast<cuuint64_t>(2) * H * kEvict * D;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), rows, static_cast<cuuint64_t>(S)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, rows * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(D), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CONVKV_OK : CONVKV_ERR_CUDA;
}

int validate(const convkv_cfg* c) {
  if (!c) return CONVKV_ERR_INVALID_ARG;
  if (c->heads < 1 || c->head_dim < 1 || c->grid_h < 1 || c->grid_w < 1 || c->first_block_frames < 1 ||
      c->block_frames < 1 || c->window_frames < 4 || c->mem_slots < 1 || c->num_states < 1 ||
      !(c->rope_theta > 0.0) || c->t_offset < 0 || c->sink_frames < 0 || c->sp_ranks < 0 ||
      c->sp_ranks > kMaxRanks || c->sp_rank < 0 || c->sp_rank >= (c->sp_ranks > 1 ? c->sp_ranks : 1))
    return CONVKV_ERR_INVALID_ARG;
  if (c->evict_frames != kEvict) return CONVKV_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return CONVKV_ERR_UNSUPPORTED;
  if (c->kv_format != CONVKV_KV_BF16 && c->kv_format != CONVKV_KV_FP8_E4M3 && c->kv_format != CONVKV_KV_NVFP4)
    return CONVKV_ERR_INVALID_ARG;
  if (c->compress_mode != CONVKV_COMPRESS_CONV && c->compress_mode != CONVKV_COMPRESS_MEAN)
    return CONVKV_ERR_INVALID_ARG;
  if (c->flags & ~(CONVKV_FLAG_DRY_RUN | CONVKV_FLAG_HOST_IO)) return CONVKV_ERR_INVALID_ARG;
  const int D = c->head_dim;
  const int dh = 2 * (D / 6);
  const bool dflt = c->rope_t == 0 && c->rope_h == 0 && c->rope_w == 0;
  if (!dflt && (c->rope_t != D - 2 * dh || c->rope_h != dh || c->rope_w != dh)) return CONVKV_ERR_UNSUPPORTED;
  const int Bmax = c->first_block_frames > c->block_frames ? c->first_block_frames : c->block_frames;
  if ((c->window_frames + Bmax) / kEvict > kMaxGroups) return CONVKV_ERR_UNSUPPORTED;
  const int64_t T = static_cast<int64_t>(c->grid_h) * c->grid_w;
  const int64_t R = c->window_frames + Bmax;
  // TMA coordinates and row counts are 32-bit
  if (T * (R > c->mem_slots ? R : c->mem_slots) > (int64_t(1) << 30) || T * Bmax > (int64_t(1) << 30) ||
      T * c->sink_frames > (int64_t(1) << 30))
    return CONVKV_ERR_UNSUPPORTED;
  // the streaming kernels index a frame's 16-byte vectors with 32-bit integers and put
  // (state, frame) pairs on the grid's y dimension
  if (T * c->heads * c->head_dim / 8 > (int64_t(1) << 30) ||
      int64_t(c->num_states) * (Bmax > c->sink_frames + c->mem_slots ? Bmax : c->sink_frames + c->mem_slots) > 65535)
    return CONVKV_ERR_UNSUPPORTED;
  const int pt = rope_pairs_t(D), ph = rope_pairs_h(D);
  const int64_t tab_units = (int64_t(c->sink_frames) + c->mem_slots + c->window_frames + Bmax) * rope_units(0, pt) +
                            int64_t(c->grid_h) * rope_units(pt, ph) + int64_t(c->grid_w) * rope_units(pt + ph, ph);
  if (tab_units * 16 > 256 * 1024) return CONVKV_ERR_UNSUPPORTED;  // RoPE tables stay cache-resident
  if (c->kv_format != CONVKV_KV_BF16 && c->compress_mode == CONVKV_COMPRESS_MEAN) return CONVKV_ERR_UNSUPPORTED;
  if (c->compress_mode == CONVKV_COMPRESS_CONV && !(c->flags & CONVKV_FLAG_DRY_RUN) && !c->conv_weight)
    return CONVKV_ERR_INVALID_ARG;
  return CONVKV_OK;
}

// Sequence shards of a block of `frames` frames: rank r holds rows [r*N/G, (r+1)*N/G).
ShardView make_view(const convkv* h, int frames) {
  ShardView v{};
  v.G = h->G;
  v.Ht = h->G * h->H;
  v.h0 = h->g * h->H;
  const int64_t N = static_cast<int64_t>(frames) * h->T;
  for (int r = 0; r <= h->G; ++r) v.off[r] = r * N / h->G;
  return v;
}

// axis with global pairs [g, g + n), positions offset .. offset+rows-1: for pair i of the
// axis the angle is pos * theta^(-2i/(2n)); units pack the pairs 2k, 2k+1 as
// (cos, cos, sin, sin), zero for a pair outside the axis
void table_axis(const convkv* h, std::vector<float4>& out, int rows, int g, int n, int64_t offset) {
  const int units = rope_units(g, n);
  for (int r = 0; r < rows; ++r)
    for (int u = 0; u < units; ++u) {
      float c[2] = {0.f, 0.f}, sn[2] = {0.f, 0.f};
      for (int q = 0; q < 2; ++q) {
        const int gp = 2 * (g / 2 + u) + q;  // global pair
        if (gp < g || gp >= g + n) continue;
        const int i = gp - g;
        const double freq = std::pow(h->cfg.rope_theta, -2.0 * i / (2.0 * n));
        const double ang = static_cast<double>(r + offset) * freq;
        c[q] = static_cast<float>(std::cos(ang));
        sn[q] = static_cast<float>(std::sin(ang));
      }
      out.push_back(make_float4(c[0], c[1], sn[0], sn[1]));
    }
}

void build_tables(const convkv* h, std::vector<float4>& out) {
  table_axis(h, out, h->tab_t_rows, 0, h->PT, h->cfg.t_offset);
  table_axis(h, out, h->gh, h->PT, h->PH, 0);
  table_axis(h, out, h->gw, h->PT + h->PH, h->PW, 0);
}

}  // namespace

extern "C" {

const char* convkv_strerror(int code) {
  switch (code) {
    case CONVKV_OK: return "ok";
    case CONVKV_ERR_INVALID_ARG: return "invalid argument";
    case CONVKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case CONVKV_ERR_BAD_ORDER: return "call out of order";
    case CONVKV_ERR_OOM: return "device allocation failed";
    case CONVKV_ERR_CUDA: return "CUDA error";
    case CONVKV_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case CONVKV_ERR_SCRATCH_LIMIT: return "request exceeds the fixed scratch area";
    default: return "unknown error";
  }
}

// Share of the last wave of `sms` SMs that a grid of `ctas` CTAs leaves idle.
static double idle_share(int64_t ctas, int sms) {
  const int64_t full = (ctas + sms - 1) / sms * sms;
  return static_cast<double>(full - ctas) / static_cast<double>(full);
}

// The group size in [1, cap] whose grid of ctas_per_state CTAs per state leaves the
// smallest share of its last wave idle.
static int wave_group(int64_t ctas_per_state, int cap, int sms) {
  int c = 1;
  double best = 2.0;
  for (int n = 1; n <= cap; ++n) {
    const double idle = idle_share(ctas_per_state * n, sms);
    if (idle < best - 1e-12) {
      best = idle;
      c = n;
    }
  }
  return c;
}

// Chunks of the host-buffer entry points.
//
// Several states: chunks of whole states.  The first chunk is one state, so the
// kernels start after one state's copy; the sizes then follow a ramp that grows 1.3
// times per chunk (1, 1, 1, 2, 2, 3, 4, ...), because a chunk's copy in has to land
// while the chunks before it compute (copying one state's K, V and queries in takes
// about 0.77 of its kernels' time at the 480x832 shape).  The steady size c (at most
// cap and 6) is the one whose attention grid, ctas_per_head * H * c CTAs, leaves the
// smallest share of its last wave idle: a chunk's kernels start only when the chunk
// before them has ended, so that idle share is lost on every chunk.  The last chunks
// shrink by thirds down to one state, so that after the last kernels only one state's
// outputs remain to copy back (a state's copy back takes about a quarter of its
// kernels' time).
//
// One state: chunks of heads, so that the copies overlap the kernels at all.  A
// chunk's attention takes whole waves: every CTA attends one query block of one head
// over all the keys, so a wave lasts as long as the CTAs themselves.  The group size
// is therefore the smallest one whose grid fills its waves to at least 85 % (one wave
// at the bench shapes: 4 heads x 32 CTAs at 512x512, 4 x 37 at 720x416, 3 x 49 at
// 480x832), else the one up to H / 2 with the fullest waves, and at least 512 bytes of
// a token row per strided copy (nh * D values); the last group takes the remaining
// heads.  Small groups start the kernels early and leave little to do and to copy
// back after the last copy in: at 512x512 the copies bound the step, at 720x416 the
// kernels, and one wave per chunk keeps the kernels dense in both.
static void plan_host_chunks(int S, int H, int D, int cap, int64_t ctas_per_head, int sms,
                             std::vector<IoChunk>& out, std::vector<IoChunk>& steady) {
  out.clear();
  steady.clear();
  if (S == 1 && H > 1) {
    const int hmax = H / 2 > 1 ? H / 2 : 1;
    int hmin = (512 + 2 * D - 1) / (2 * D);
    if (hmin > hmax) hmin = hmax;
    int hg = hmin;
    double best = -1.0;
    for (int n = hmin; n <= hmax; ++n) {
      const double fill = 1.0 - idle_share(ctas_per_head * n, sms);
      if (fill >= 0.85) {
        hg = n;
        break;
      }
      if (fill > best + 1e-12) {
        best = fill;
        hg = n;
      }
    }
    for (int h0 = 0; h0 < H; h0 += hg) out.push_back({0, 1, h0, H - h0 < hg ? H - h0 : hg});
    steady = out;
    return;
  }
  const int c = wave_group(ctas_per_head * H, cap < 6 ? (cap > 0 ? cap : 1) : 6, sms);
  std::vector<int> tail;
  for (int t = c; t > 1;) {
    t = (t + 2) / 3;
    tail.push_back(t);
  }
  int tail_states = 0;
  for (int t : tail) tail_states += t;
  if (tail_states >= S) tail.clear(), tail_states = 0;
  int g0 = 0;
  for (int n100 = 100; g0 < S - tail_states; n100 = n100 * 130 / 100) {
    int n = n100 / 100;
    if (n > c) n = c;
    if (n > S - tail_states - g0) n = S - tail_states - g0;
    out.push_back({g0, n, 0, H});
    g0 += n;
  }
  for (int t : tail) {
    out.push_back({g0, t, 0, H});
    g0 += t;
  }
  // queued steps: their copies in run ahead during the previous step, so neither the
  // ramp nor the short tail is needed, and fewer launch boundaries are better: chunks
  // of up to cap states, at least two per step so that the next step's first chunk
  // can be copied in while this step's later chunks compute
  const int cs = cap < (S + 1) / 2 ? cap : (S + 1) / 2;
  for (int s0 = 0; s0 < S; s0 += cs) steady.push_back({s0, S - s0 < cs ? S - s0 : cs, 0, H});
}

// Copy streams and events of the host-buffer entry points, and their chunk plan.
static int create_host_io(convkv_t* h) {
  plan_host_chunks(h->S, h->H, h->D, h->fp8 ? h->Sg : h->S, h->ctas_per_head(), h->sms, h->io_plan[0],
                   h->io_plan[1]);
  h->io_nmax = static_cast<int>(std::max(h->io_plan[0].size(), h->io_plan[1].size()));
  if (cudaStreamCreateWithFlags(&h->io_in, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&h->io_back, cudaStreamNonBlocking) != cudaSuccess)
    return CONVKV_ERR_CUDA;
  h->io_ev.assign(3 * static_cast<size_t>(h->io_nmax), nullptr);
  for (auto& ev : h->io_ev)
    if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return CONVKV_ERR_CUDA;
  return CONVKV_OK;
}

static void release_host_io(convkv_t* h) {
  if (h->io_in) cudaStreamSynchronize(h->io_in);
  if (h->io_back) cudaStreamSynchronize(h->io_back);
  for (auto& ev : h->io_ev)
    if (ev) cudaEventDestroy(ev);
  h->io_ev.clear();
  if (h->io_in) cudaStreamDestroy(h->io_in);
  if (h->io_back) cudaStreamDestroy(h->io_back);
  h->io_in = h->io_back = nullptr;
}

int convkv_create(const convkv_cfg* cfg, convkv_t** out) {
  if (!out) return CONVKV_ERR_INVALID_ARG;
  *out = nullptr;
  int rc = validate(cfg);
  if (rc) return rc;
  convkv* h = new (std::nothrow) convkv;
  if (!h) return CONVKV_ERR_OOM;
  h->cfg = *cfg;
  h->H = cfg->heads;
  h->D = cfg->head_dim;
  h->gh = cfg->grid_h;
  h->gw = cfg->grid_w;
  h->T = cfg->grid_h * cfg->grid_w;
  h->b1 = cfg->first_block_frames;
  h->bn = cfg->block_frames;
  h->Bmax = h->b1 > h->bn ? h->b1 : h->bn;
  h->W = cfg->window_frames;
  h->C = cfg->mem_slots;
  h->R = h->W + h->Bmax;
  h->S = cfg->num_states;
  h->PH = cfg->head_dim / 6;
  h->PW = h->PH;
  h->PT = (cfg->head_dim - 4 * h->PH) / 2;
  h->Rs = cfg->sink_frames;
  h->G = cfg->sp_ranks > 1 ? cfg->sp_ranks : 1;
  h->g = cfg->sp_rank;
  h->tab_t_rows = h->Rs + h->C + h->W + h->Bmax;
  h->dry = (cfg->flags & CONVKV_FLAG_DRY_RUN) != 0;
  h->host_io = (cfg->flags & CONVKV_FLAG_HOST_IO) != 0;
  h->mean = cfg->compress_mode == CONVKV_COMPRESS_MEAN;
  h->fp8 = cfg->kv_format != CONVKV_KV_BF16;
  h->fp4 = cfg->kv_format == CONVKV_KV_NVFP4;
  h->prerot = !h->fp8;
  h->stream = static_cast<cudaStream_t>(cfg->stream);
  h->cfg.conv_weight = nullptr;
  // e4m3 / NVFP4: the dequantisation scratch holds up to 4 GiB of states at a time
  if (h->fp8) {
    const size_t per_state = static_cast<size_t>(h->C + h->W) * h->frame_elems() * 2 * 2;
    const size_t budget = size_t(4) << 30;
    h->Sg = static_cast<int>(per_state * h->S <= budget ? h->S : (budget / per_state > 0 ? budget / per_state : 1));
  }
  if (!h->dry) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || h->sms < 1) {
      delete h;
      return CONVKV_ERR_CUDA;
    }
  }
  if (h->dry) {
    // the host-buffer chunk plan only, for a B200's 148 SMs (no device is queried)
    if (h->host_io)
      plan_host_chunks(h->S, h->H, h->D, h->fp8 ? h->Sg : h->S, h->ctas_per_head(), h->sms, h->io_plan[0],
                       h->io_plan[1]);
    *out = h;
    return CONVKV_OK;
  }

  const size_t fe = static_cast<size_t>(h->frame_elems());
  // bytes of one cached frame: bf16 2 per element, e4m3 1, NVFP4 1/2 (+ 1/16 of block scales)
  const size_t fbytes = h->fp4 ? fe / 2 : (h->fp8 ? fe : 2 * fe);
  const size_t ring_b = static_cast<size_t>(h->S) * h->R * fbytes;
  const size_t mem_b = static_cast<size_t>(h->S) * h->C * fbytes;
  const size_t rbs_b = h->fp4 ? static_cast<size_t>(h->S) * h->R * fe / 16 : 0;
  const size_t mbs_b = h->fp4 ? static_cast<size_t>(h->S) * h->C * fe / 16 : 0;
  const size_t rsc_b = h->fp8 ? static_cast<size_t>(h->S) * 2 * h->R * h->H * sizeof(float) : 0;
  const size_t msc_b = h->fp8 ? static_cast<size_t>(h->S) * 2 * h->C * h->H * sizeof(float) : 0;
  const size_t stg_b = h->fp8 ? static_cast<size_t>(h->S) * h->Bmax * fe * 2 : 0;
  const size_t amax_n = static_cast<size_t>(h->S) * 2 * h->H * (h->Bmax > kMaxGroups ? h->Bmax : kMaxGroups);
  const size_t amax_b = h->fp8 ? amax_n * sizeof(unsigned int) : 0;
  const size_t w_b = h->mean ? 0 : static_cast<size_t>(h->S) * 2 * h->H * kEvict * h->D * h->D * 2;
  std::vector<float4> tab;
  build_tables(h, tab);
  const size_t tab_b = tab.size() * sizeof(float4);
  const size_t io_b = h->host_io ? static_cast<size_t>(h->S) * h->Bmax * fe * 2 : 0;
  const size_t sink_b = static_cast<size_t>(h->S) * h->Rs * fe * 2;
  const size_t rkr_b = h->prerot ? ring_b : 0;
  const size_t mkr_b = h->prerot ? mem_b : 0;
  const size_t scr_b = h->fp8 ? static_cast<size_t>(h->Sg) * (h->C + h->W) * fe * 2 : 0;
  // e4m3 / NVFP4: the conv's fp32 outputs for the groups of one append (the window
  // holds at most W + Bmax frames before an append's evictions, so at most
  // ceil(Bmax / 5) groups)
  h->gmax = (h->Bmax + kEvict - 1) / kEvict;
  const size_t acc_b = h->fp8 ? static_cast<size_t>(h->S) * h->gmax * 2 * fe * sizeof(float) : 0;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t o_rk = take(ring_b), o_rv = take(ring_b), o_mk = take(mem_b), o_mv = take(mem_b), o_w = take(w_b),
               o_tab = take(tab_b), o_st = take(sizeof(int)), o_q = take(io_b), o_k = take(io_b),
               o_v = take(io_b), o_o = take(io_b), o_rsc = take(rsc_b), o_msc = take(msc_b), o_sk = take(stg_b),
               o_sv = take(stg_b), o_am = take(amax_b), o_rfk = take(sink_b), o_rfv = take(sink_b),
               o_rbk = take(rbs_b), o_rbv = take(rbs_b), o_mbk = take(mbs_b), o_mbv = take(mbs_b),
               o_rkr = take(rkr_b), o_mkr = take(mkr_b), o_skr = take(sink_b), o_sck = take(scr_b),
               o_scv = take(scr_b), o_acc = take(acc_b);
  h->arena_bytes = off;
  cudaError_t e = cudaMalloc(&h->arena, h->arena_bytes);
  if (e != cudaSuccess) {
    h->arena = nullptr;
    delete h;
    cudaGetLastError();
    return CONVKV_ERR_OOM;
  }
  char* a = static_cast<char*>(h->arena);
  h->ringK = a + o_rk;
  h->ringV = a + o_rv;
  h->memK = a + o_mk;
  h->memV = a + o_mv;
  h->weights = w_b ? a + o_w : nullptr;
  h->tables = reinterpret_cast<float4*>(a + o_tab);
  h->status = reinterpret_cast<int*>(a + o_st);
  if (h->fp8) {
    h->ring_scale = reinterpret_cast<float*>(a + o_rsc);
    h->mem_scale = reinterpret_cast<float*>(a + o_msc);
    h->stageK = a + o_sk;
    h->stageV = a + o_sv;
    h->amax = reinterpret_cast<unsigned int*>(a + o_am);
    h->scrK = a + o_sck;
    h->scrV = a + o_scv;
    h->convacc = reinterpret_cast<float*>(a + o_acc);
  }
  if (h->fp4) {
    h->ringBK = reinterpret_cast<uint8_t*>(a + o_rbk);
    h->ringBV = reinterpret_cast<uint8_t*>(a + o_rbv);
    h->memBK = reinterpret_cast<uint8_t*>(a + o_mbk);
    h->memBV = reinterpret_cast<uint8_t*>(a + o_mbv);
  }
  if (h->prerot) {
    h->ringKr = a + o_rkr;
    h->memKr = a + o_mkr;
  }
  if (h->Rs) {
    h->sinkK = a + o_rfk;
    h->sinkV = a + o_rfv;
    h->sinkKr = a + o_skr;
  }
  if (h->host_io) {
    h->io_q = a + o_q;
    h->io_k = a + o_k;
    h->io_v = a + o_v;
    h->io_out = a + o_o;
  }
  // zero fill: rows past a segment's end are read (then masked) and must be finite
  if ((e = cudaMemsetAsync(h->arena, 0, h->arena_bytes, h->stream)) != cudaSuccess) goto fail_cuda;
  if ((e = cudaMemcpyAsync(h->tables, tab.data(), tab_b, cudaMemcpyHostToDevice, h->stream)) != cudaSuccess)
    goto fail_cuda;
  if (w_b) {
    if ((e = static_cast<cudaError_t>(launch_permute_weights(cfg->conv_weight, h->weights, h->S, h->H, h->D,
                                                             h->stream))) != cudaSuccess)
      goto fail_cuda;
    h->launches++;
  }
  if ((e = cudaStreamSynchronize(h->stream)) != cudaSuccess) goto fail_cuda;
  if (h->fp8) {
    // the conv stages the ring's code tiles with TMA; the attention reads the bf16
    // staging of the current block and the dequantisation scratch
    const int cb = h->fp4 ? h->D / 2 : h->D;
    rc = encode_4d(&h->mapStageK, h->stageK, h->D, h->H, static_cast<int64_t>(h->Bmax) * h->T, h->S);
    if (!rc) rc = encode_4d(&h->mapStageV, h->stageV, h->D, h->H, static_cast<int64_t>(h->Bmax) * h->T, h->S);
    if (!rc) rc = encode_codes(&h->mapRingCK, h->ringK, cb, h->H, static_cast<int64_t>(h->R) * h->T, h->S);
    if (!rc) rc = encode_codes(&h->mapRingCV, h->ringV, cb, h->H, static_cast<int64_t>(h->R) * h->T, h->S);
    const int64_t scr_rows = static_cast<int64_t>(h->C + h->W) * h->T;
    if (!rc) rc = encode_4d(&h->mapScrK, h->scrK, h->D, h->H, scr_rows, h->Sg);
    if (!rc) rc = encode_4d(&h->mapScrV, h->scrV, h->D, h->H, scr_rows, h->Sg);
  } else {
    rc = encode_4d(&h->mapRingK, h->ringK, h->D, h->H, static_cast<int64_t>(h->R) * h->T, h->S);
    if (!rc) rc = encode_4d(&h->mapRingKr, h->ringKr, h->D, h->H, static_cast<int64_t>(h->R) * h->T, h->S);
    if (!rc) rc = encode_4d(&h->mapRingV, h->ringV, h->D, h->H, static_cast<int64_t>(h->R) * h->T, h->S);
    if (!rc) rc = encode_4d(&h->mapMemK, h->memK, h->D, h->H, static_cast<int64_t>(h->C) * h->T, h->S);
    if (!rc) rc = encode_4d(&h->mapMemV, h->memV, h->D, h->H, static_cast<int64_t>(h->C) * h->T, h->S);
    if (!rc) rc = encode_4d(&h->mapMemKr, h->memKr, h->D, h->H, static_cast<int64_t>(h->C) * h->T, h->S);
  }
  if (!rc && h->Rs) rc = encode_4d(&h->mapSinkKr, h->sinkKr, h->D, h->H, static_cast<int64_t>(h->Rs) * h->T, h->S);
  if (!rc && h->Rs) rc = encode_4d(&h->mapSinkK, h->sinkK, h->D, h->H, static_cast<int64_t>(h->Rs) * h->T, h->S);
  if (!rc && h->Rs) rc = encode_4d(&h->mapSinkV, h->sinkV, h->D, h->H, static_cast<int64_t>(h->Rs) * h->T, h->S);
  if (!rc && w_b) rc = encode_weights(&h->mapW, h->weights, h->D, h->H, h->S);
  if (!rc && h->host_io) rc = create_host_io(h);
  if (rc) {
    release_host_io(h);
    cudaFree(h->arena);
    delete h;
    return rc;
  }
  *out = h;
  return CONVKV_OK;
fail_cuda:
  cudaStreamSynchronize(h->stream);
  cudaFree(h->arena);
  delete h;
  return CONVKV_ERR_CUDA;
}

void convkv_destroy(convkv_t* h) {
  if (!h) return;
  if (h->arena) {
    cudaStreamSynchronize(h->stream);
    release_host_io(h);
    cudaFree(h->arena);
  }
  delete h;
}

size_t convkv_state_bytes(const convkv_t* h) { return h ? h->arena_bytes : 0; }

int64_t convkv_launch_count(const convkv_t* h) { return h ? h->launches : 0; }

int convkv_last_cuda_error(const convkv_t* h) { return h ? h->last_cuda : 0; }

// Rotated copies of the reference frames and memory slots for the time table of the
// step (base B0): RoPE Reset moves their positions with every eviction, so they are
// rotated again whenever B0 moves, or the reference frames were given anew.
static int rotate_moving_keys(convkv_t* h, int64_t B0) {
  RotateParams rp{};
  rp.S = h->S;
  rp.r = h->Rs;
  rp.m = h->prerot ? h->m() : 0;
  rp.C = h->C;
  rp.pos0 = static_cast<int>((h->Sn - h->m()) % h->C);
  rp.frame_vecs = h->frame_elems() / 8;
  rp.H = h->H;
  rp.grid_w = h->gw;
  rp.sink_src = h->sinkK;
  rp.sink_dst = h->sinkKr;
  rp.mem_src = h->memK;
  rp.mem_dst = h->memKr;
  rp.tables = h->tables;
  rp.tab_t_rows = h->tab_t_rows;
  rp.tab_h_rows = h->gh;
  rp.div_heads = FastDiv(static_cast<uint32_t>(h->H));
  rp.div_grid_w = FastDiv(static_cast<uint32_t>(h->gw));
  const int e = launch_rotate_keys(h->D, rp, h->stream);
  if (e) return h->cuda_fail(static_cast<cudaError_t>(e));
  if (rp.r + rp.m > 0) h->launches++;
  h->rot_B0 = B0;
  h->rot_sink_stale = false;
  return CONVKV_OK;
}

// The steps of one append.  Advances the counters first (the launches read the new
// ones); append_impl restores them when a step fails.
// The ring append's parameters for states [g0, g0 + n): every per-state buffer moves
// by g0 states (the kernels index states from 0).
static AppendParams states_slice(const convkv_t* h, const AppendParams& a, int g0, int n, int frames) {
  if (g0 == 0 && n == a.S) return a;
  AppendParams p = a;
  p.S = n;
  const int64_t fe = h->frame_elems();
  const int64_t g = g0;
  if (p.ringKr) p.ringKr = static_cast<char*>(p.ringKr) + g * h->R * fe * 2;
  if (h->fp8) {
    const int64_t code_bytes = h->fp4 ? fe / 2 : fe;  // per frame
    p.amax += g * 2 * frames * h->H;
    p.ring8[0] += g * h->R * code_bytes;
    p.ring8[1] += g * h->R * code_bytes;
    p.ring_scale += g * 2 * h->R * h->H;
    if (h->fp4) {
      p.ring_bs[0] += g * h->R * (fe / 16);
      p.ring_bs[1] += g * h->R * (fe / 16);
    }
    p.stage[0] = static_cast<char*>(p.stage[0]) + g * h->Bmax * fe * 2;
    p.stage[1] = static_cast<char*>(p.stage[1]) + g * h->Bmax * fe * 2;
  }
  return p;
}

// Step 4 of the append for the states and heads of chunk `ck`: the new block into the
// ring (and the rotated K / the staging copy).  With host buffers arriving by chunks
// (c >= 0: the chunk's index), it first waits for the chunk's copy.
static int ring_append_chunk(convkv_t* h, const AppendParams& ap, const void* k, const void* v, const IoChunk& ck,
                             int c) {
  if (c >= 0) {
    cudaError_t w = cudaStreamWaitEvent(h->stream, h->ev_in(c), 0);
    if (w != cudaSuccess) return h->cuda_fail(w);
  }
  const int frames = ap.b, g0 = ck.g0;
  AppendParams a = states_slice(h, ap, g0, ck.n, frames);
  a.h0 = ck.h0;
  a.nh = ck.nh;
  a.div_nh = FastDiv(static_cast<uint32_t>(ck.nh));
  const int64_t in_off = static_cast<int64_t>(g0) * frames * h->frame_elems() * 2;
  const void* kc = k ? static_cast<const char*>(k) + in_off : nullptr;
  const void* vc = v ? static_cast<const char*>(v) + in_off : nullptr;
  int e;
  if (h->fp8) {
    e = launch_append_fp8(a, kc, vc, h->stream);
    h->launches += 2;
  } else {
    const int64_t ring_off = static_cast<int64_t>(g0) * h->R * h->frame_elems() * 2;
    e = launch_append_bf16(a, kc, vc, static_cast<char*>(h->ringK) + ring_off, static_cast<char*>(h->ringV) + ring_off,
                           h->stream);
    h->launches++;
  }
  if (e) return h->cuda_fail(static_cast<cudaError_t>(e));
  // the chunk's k / v staging is free for the next call once these kernels are done
  if (c >= 0) {
    cudaError_t w = cudaEventRecord(h->ev_done(c), h->stream);
    if (w != cudaSuccess) return h->cuda_fail(w);
  }
  return CONVKV_OK;
}

static int append_steps(convkv_t* h, const void* k, const void* v, const void* const* k_sh,
                        const void* const* v_sh, int frames) {
  // 1. the previous current block joins the window
  h->P += h->bcur;
  // 2. evict groups of 5 while the window holds more than W frames
  std::vector<std::pair<int64_t, int64_t>> groups;  // (first frame, slot index)
  while (h->P - h->E > h->W) {
    groups.emplace_back(h->E, h->Sn);
    h->E += kEvict;
    h->Sn += 1;
  }
  h->last_groups = static_cast<int>(groups.size());
  // groups older than the last C of this call would be dropped by the FIFO before anyone reads them
  const size_t first = groups.size() > static_cast<size_t>(h->C) ? groups.size() - h->C : 0;
  h->bcur = frames;
  h->blocks += 1;

  if (groups.size() > first) {
    if (cudaError_t g = h->step_gate()) return h->cuda_fail(g);
    if (!h->dry) {
      ConvParams cp{};
      cp.H = h->H;
      cp.T = h->T;
      cp.S = h->S;
      cp.C = h->C;
      cp.R = h->R;
      cp.ngroups = static_cast<int>(groups.size() - first);
      for (size_t g = first; g < groups.size(); ++g) {
        ConvGroup& cg = cp.grp[g - first];
        for (int j = 0; j < kEvict; ++j) cg.ring_slot[j] = static_cast<int>((groups[g].first + j) % h->R);
        cg.mem_pos = static_cast<int>(groups[g].second % h->C);
      }
      cp.memK = h->memK;
      cp.memV = h->memV;
      cp.status = h->status;
      int e;
      if (h->fp8) {
        cp.ring8[0] = static_cast<const uint8_t*>(h->ringK);
        cp.ring8[1] = static_cast<const uint8_t*>(h->ringV);
        cp.ring_scale = h->ring_scale;
        cp.amax = h->amax;
        cp.acc = h->convacc;
        cp.mem_scale = h->mem_scale;
        if (cp.ngroups > h->gmax) return h->cuda_fail(cudaErrorInvalidValue);
        cp.ring_bs[0] = h->ringBK;
        cp.ring_bs[1] = h->ringBV;
        cp.mem_bs[0] = h->memBK;
        cp.mem_bs[1] = h->memBV;
        e = h->fp4 ? launch_conv_fp4(h->D, cp, h->mapRingCK, h->mapRingCV, h->mapW, h->stream)
                   : launch_conv_fp8(h->D, cp, h->mapRingCK, h->mapRingCV, h->mapW, h->stream);
        h->launches += 2;
      } else {
        e = h->mean ? launch_mean_bf16(h->D, cp, h->ringK, h->ringV, h->stream)
                    : launch_conv_bf16(h->D, cp, h->mapRingK, h->mapRingV, h->mapW, h->stream);
        h->launches++;
      }
      if (e) return h->cuda_fail(static_cast<cudaError_t>(e));
    }
  }
  // 3. the time table of this step: absolute positions B0 + i, B0 = E - r - m (+ t_offset)
  const int64_t B0 = h->E - h->Rs - h->m() + h->cfg.t_offset;
  if (cudaError_t g = h->step_gate()) return h->cuda_fail(g);
  if (!h->dry) {
    h->tab_t_host.clear();
    table_axis(h, h->tab_t_host, h->tab_t_rows, 0, h->PT, B0);
    cudaError_t e = cudaMemcpyAsync(h->tables, h->tab_t_host.data(), h->tab_t_host.size() * sizeof(float4),
                                    cudaMemcpyHostToDevice, h->stream);
    if (e != cudaSuccess) return h->cuda_fail(e);
  }
  // 3b. memory slots (bf16 format) and reference frames rotated for this table
  if ((h->prerot || h->Rs) && (B0 != h->rot_B0 || h->rot_sink_stale)) {
    if (cudaError_t g = h->step_gate()) return h->cuda_fail(g);
    if (!h->dry) {
      if (int rc = rotate_moving_keys(h, B0)) return rc;
    } else {
      h->rot_B0 = B0;
      h->rot_sink_stale = false;
    }
  }
  // 4. the new block becomes the current block: copy into ring slots (P + f) mod R
  if (cudaError_t g = h->step_gate()) return h->cuda_fail(g);
  if (h->dry) return CONVKV_OK;
  AppendParams ap{};
  ap.S = h->S;
  ap.b = frames;
  ap.R = h->R;
  ap.slot0 = static_cast<int>(h->P % h->R);
  ap.frame_elems = h->frame_elems();
  ap.H = h->H;
  ap.D = h->D;
  ap.div_heads = FastDiv(static_cast<uint32_t>(h->H));
  ap.div_grid_w = FastDiv(static_cast<uint32_t>(h->gw));
  if (h->prerot || h->fp8) {
    // bf16: K is also written rotated into ringKr; e4m3 / NVFP4: the current block's
    // bf16 staging copy of K is written rotated
    ap.ringKr = h->prerot ? h->ringKr : nullptr;
    ap.tables = h->tables;
    ap.tab_t_rows = h->tab_t_rows;
    ap.tab_h_rows = h->gh;
    ap.t_row0 = h->Rs + h->m() + h->w();
    ap.grid_w = h->gw;
  }
  if (k_sh) {
    ap.sv = make_view(h, frames);
    for (int r = 0; r < h->G; ++r) {
      ap.k_sh[r] = k_sh[r];
      ap.v_sh[r] = v_sh[r];
    }
  }
  if (h->fp8) {
    ap.amax = h->amax;
    ap.ring8[0] = static_cast<uint8_t*>(h->ringK);
    ap.ring8[1] = static_cast<uint8_t*>(h->ringV);
    ap.ring_scale = h->ring_scale;
    ap.ring_bs[0] = h->ringBK;
    ap.ring_bs[1] = h->ringBV;
    ap.fp4 = h->fp4 ? 1 : 0;
    ap.stage[0] = h->stageK;
    ap.stage[1] = h->stageV;
    ap.stage_frames = h->Bmax;
  }
  if (h->io_defer) {
    h->io_ap = ap;
    return CONVKV_OK;
  }
  // one launch set for all states and heads, or (host buffers arriving chunk by chunk)
  // one per chunk, each after its chunk's copy
  if (!h->io_pending) return ring_append_chunk(h, ap, k, v, IoChunk{0, h->S, 0, h->H}, -1);
  for (int c = 0; c < h->io_nchunks; ++c)
    if (int rc = ring_append_chunk(h, ap, k, v, h->io_chunks[c], c)) return rc;
  return CONVKV_OK;
}

// One append, all or nothing on the host side: when a launch step fails, the
// counters go back to their values before the call.  A conv that already ran for
// the call may have rewritten a memory position (with the new slot, made from ring
// frames that no later step of the call touches), so until an append succeeds the
// handle refuses attends; the next append recomputes that slot from the same frames.
static int append_impl(convkv_t* h, const void* k, const void* v, const void* const* k_sh,
                       const void* const* v_sh, int frames) {
  const int64_t P = h->P, E = h->E, Sn = h->Sn, blocks = h->blocks;
  const int bcur = h->bcur, last_groups = h->last_groups;
  h->steps = 0;
  const int rc = append_steps(h, k, v, k_sh, v_sh, frames);
  h->need_append = rc != CONVKV_OK;
  if (rc != CONVKV_OK) {
    h->P = P;
    h->E = E;
    h->Sn = Sn;
    h->blocks = blocks;
    h->bcur = bcur;
    h->last_groups = last_groups;
  }
  return rc;
}

int convkv_debug_fail_step(convkv_t* h, int step) {
  if (!h || step < -1) return CONVKV_ERR_INVALID_ARG;
  h->fail_at = step;
  return CONVKV_OK;
}

int convkv_append_block(convkv_t* h, const void* k, const void* v, int frames) {
  if (!h || frames < 1 || frames > h->Bmax) return CONVKV_ERR_INVALID_ARG;
  if (!h->dry && (!k || !v)) return CONVKV_ERR_INVALID_ARG;
  return append_impl(h, k, v, nullptr, nullptr, frames);
}

static bool shards_ok(const convkv_t* h, const void* const* a, const void* const* b) {
  if (!a || !b) return false;
  for (int r = 0; r < h->G; ++r)
    if (!a[r] || !b[r]) return false;
  return true;
}

int convkv_append_block_sp(convkv_t* h, const void* const* k_shards, const void* const* v_shards, int frames) {
  if (!h || h->G < 2 || frames < 1 || frames > h->Bmax) return CONVKV_ERR_INVALID_ARG;
  if (!h->dry && !shards_ok(h, k_shards, v_shards)) return CONVKV_ERR_INVALID_ARG;
  return append_impl(h, nullptr, nullptr, h->dry ? nullptr : k_shards, h->dry ? nullptr : v_shards, frames);
}

int convkv_set_sink(convkv_t* h, const void* k, const void* v) {
  if (!h || (!h->dry && (!k || !v))) return CONVKV_ERR_INVALID_ARG;
  if (h->Rs == 0) return CONVKV_ERR_BAD_ORDER;
  if (!h->dry) {
    const size_t bytes = static_cast<size_t>(h->S) * h->Rs * h->frame_elems() * 2;
    cudaError_t e = cudaMemcpyAsync(h->sinkK, k, bytes, cudaMemcpyDeviceToDevice, h->stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(h->sinkV, v, bytes, cudaMemcpyDeviceToDevice, h->stream);
    if (e != cudaSuccess) return h->cuda_fail(e);
  }
  h->rot_sink_stale = true;
  // after the first append the step's table exists: rotate the new frames now (before
  // that, the first append does it)
  if (h->blocks > 0 && !h->need_append) {
    if (!h->dry) {
      if (int rc = rotate_moving_keys(h, h->rot_B0)) return rc;
    } else {
      h->rot_sink_stale = false;
    }
  }
  h->sink_set = true;
  return CONVKV_OK;
}

// Copy of chunk ck's rows of a [S][rows][H][D] bf16 tensor (bps bytes per state)
// between host and device: one contiguous copy for whole states, a strided one (one
// row of nh * D values per token) for a head range.
static cudaError_t copy_chunk(const convkv_t* h, const IoChunk& ck, void* dst, const void* src, size_t bps,
                              cudaMemcpyKind kind, cudaStream_t st) {
  const size_t off = static_cast<size_t>(ck.g0) * bps;
  if (ck.nh == h->H)
    return cudaMemcpyAsync(static_cast<char*>(dst) + off, static_cast<const char*>(src) + off, ck.n * bps, kind, st);
  const size_t row = static_cast<size_t>(h->H) * h->D * 2;
  const size_t col = static_cast<size_t>(ck.h0) * h->D * 2;
  return cudaMemcpy2DAsync(static_cast<char*>(dst) + off + col, row, static_cast<const char*>(src) + off + col, row,
                           static_cast<size_t>(ck.nh) * h->D * 2, bps / row, kind, st);
}

// out_host: the host-buffer form (queries copied in by chunks, see
// convkv_attend_host); each chunk's attention waits for its queries, and its outputs
// are copied back to out_host as soon as it ends.  [cbeg, cend): the chunks attended
// by this call.
static int attend_impl(convkv_t* h, const void* q, void* out, const void* const* q_sh, void* const* o_sh,
                       char* out_host = nullptr, int cbeg = 0, int cend = -1) {
  const int r = h->Rs, m = h->m(), w = h->w(), b = h->bcur, T = h->T;
  AttnParams ap{};
  ap.H = h->H;
  ap.T = T;
  ap.grid_w = h->gw;
  ap.Nq = b * T;
  ap.tq0 = r + m + w;
  int tiles = 0;
  // every key segment is bf16 and stored rotated: the ring's rotated K (window and
  // current, bf16 format), the rotated memory and reference frames, the dequantised
  // scratch and the rotated staging of the current block (e4m3 / NVFP4 formats)
  auto add = [&](int buf, int frame0, int nframes, int local) {
    KeySeg& s = ap.seg[ap.nseg++];
    s.buf = buf;
    s.row0 = frame0 * T;
    s.nrows = nframes * T;
    s.local = local;
    tiles += (s.nrows + 127) / 128;
  };
  if (r > 0) add(3, 0, r, 0);
  if (h->fp8) {
    // [memory | window] dequantised into the scratch in attend order, then the
    // current block's bf16 staging
    if (m + w > 0) add(0, 0, m + w, 1);
    add(2, 0, b, 0);
  } else {
    if (m > 0) {
      const int pos0 = static_cast<int>((h->Sn - m) % h->C);
      const int n1 = m < h->C - pos0 ? m : h->C - pos0;
      add(1, pos0, n1, 0);
      if (m > n1) add(1, 0, m - n1, 0);
    }
    // window and current block are consecutive ring frames
    const int n = w + b;
    const int start = static_cast<int>(h->E % h->R);
    const int n1 = n < h->R - start ? n : h->R - start;
    if (n1 > 0) add(0, start, n1, 0);
    if (n > n1) add(0, 0, n - n1, 0);
  }
  ap.ntiles = tiles;
  ap.tab_t_rows = h->tab_t_rows;
  ap.tab_h_rows = h->gh;
  ap.tab_w_rows = h->gw;
  ap.tables = h->tables;
  ap.out = static_cast<__nv_bfloat16*>(out);
  ap.q_scale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(h->D)));
  ap.status = h->status;
  CUtensorMap mq{};
  if (q_sh) {
    // queries are gathered from the sequence shards by the kernel: no TMA map for them
    ap.sv = make_view(h, b);
    for (int r = 0; r < h->G; ++r) {
      ap.q_sh[r] = static_cast<const __nv_bfloat16*>(q_sh[r]);
      ap.o_sh[r] = static_cast<__nv_bfloat16*>(o_sh[r]);
    }
  } else {
    int rc = encode_4d(&mq, const_cast<void*>(q), h->D, h->H, ap.Nq, h->S);
    if (rc) return rc;
  }
  CUtensorMap km[4], vm[4];
  if (h->fp8) {
    km[0] = h->mapScrK; km[1] = h->mapScrK; km[2] = h->mapStageK;
    vm[0] = h->mapScrV; vm[1] = h->mapScrV; vm[2] = h->mapStageV;
  } else {
    km[0] = h->mapRingKr; km[1] = h->mapMemKr; km[2] = h->mapRingK;
    vm[0] = h->mapRingV; vm[1] = h->mapMemV; vm[2] = h->mapRingV;
  }
  km[3] = r ? h->mapSinkKr : km[2];
  vm[3] = r ? h->mapSinkV : vm[2];
  const size_t bps = static_cast<size_t>(b) * h->frame_elems() * 2;   // query / output bytes per state
  // before chunk c's attention: wait for its queries; after it: send its outputs back
  // (and for the previous call's copy back of the chunk's output staging)
  auto io_before = [&](int c) -> cudaError_t {
    if (c < 0) return cudaSuccess;
    cudaError_t e = cudaStreamWaitEvent(h->stream, h->ev_in(c), 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->stream, h->ev_out(h->io_prev(c, b)), 0);
    return e;
  };
  auto io_after = [&](int c) -> cudaError_t {
    if (c < 0) return cudaSuccess;
    cudaError_t e = cudaEventRecord(h->ev_done(c), h->stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->io_back, h->ev_done(c), 0);
    if (e == cudaSuccess) e = copy_chunk(h, h->io_chunks[c], out_host, out, bps, cudaMemcpyDeviceToHost, h->io_back);
    if (e == cudaSuccess) e = cudaEventRecord(h->ev_out(c), h->io_back);
    return e;
  };
  // the launches: the host-buffer chunks [cbeg, cend) (index c), else all states at
  // once (bf16) or groups of Sg states (the scratch's capacity), with every head.
  // Groups are as large as they can be: every launch boundary leaves SMs idle while
  // the last CTAs of a launch finish (groups of 4 states, whose last wave is fuller
  // than that of groups of 7, measured 0.45 % slower at 480x832 x 40 states)
  struct Unit {
    IoChunk ck;
    int c;
  };
  std::vector<Unit> units;
  if (out_host) {
    if (cend < 0) cend = h->io_nchunks;
    for (int c = cbeg; c < cend; ++c) units.push_back({h->io_chunks[c], c});
  } else {
    const int step = h->fp8 ? h->Sg : h->S;
    for (int g0 = 0; g0 < h->S; g0 += step) units.push_back({{g0, h->S - g0 < step ? h->S - g0 : step, 0, h->H}, -1});
  }
  if (!h->fp8) {
    for (const Unit& u : units) {
      if (cudaError_t w = io_before(u.c)) return h->cuda_fail(w);
      ap.state0 = u.ck.g0;
      ap.head0 = u.ck.h0;
      ap.nheads = u.ck.nh;
      int e = launch_attend(h->D, ap, mq, km, vm, u.ck.n, h->stream);
      h->launches++;
      if (e) return h->cuda_fail(static_cast<cudaError_t>(e));
      if (cudaError_t w = io_after(u.c)) return h->cuda_fail(w);
    }
    return CONVKV_OK;
  }
  // e4m3 / NVFP4: per group of states, dequantise [memory | window] into the scratch
  // (K rotated), then attend over [reference | scratch | staging]
  DequantParams dp{};
  dp.m = m;
  dp.w = w;
  dp.r = r;
  dp.C = h->C;
  dp.R = h->R;
  dp.H = h->H;
  dp.grid_w = h->gw;
  dp.pos0 = static_cast<int>((h->Sn - m) % h->C);
  dp.ring0 = static_cast<int>(h->E % h->R);
  dp.out_frames = h->C + h->W;
  dp.fp4 = h->fp4 ? 1 : 0;
  dp.frame_elems = h->frame_elems();
  dp.ring8[0] = static_cast<const uint8_t*>(h->ringK);
  dp.ring8[1] = static_cast<const uint8_t*>(h->ringV);
  dp.mem8[0] = static_cast<const uint8_t*>(h->memK);
  dp.mem8[1] = static_cast<const uint8_t*>(h->memV);
  dp.ring_scale = h->ring_scale;
  dp.mem_scale = h->mem_scale;
  dp.ring_bs[0] = h->ringBK;
  dp.ring_bs[1] = h->ringBV;
  dp.mem_bs[0] = h->memBK;
  dp.mem_bs[1] = h->memBV;
  dp.out[0] = h->scrK;
  dp.out[1] = h->scrV;
  dp.tables = h->tables;
  dp.tab_t_rows = h->tab_t_rows;
  dp.tab_h_rows = h->gh;
  dp.div_heads = FastDiv(static_cast<uint32_t>(h->H));
  dp.div_grid_w = FastDiv(static_cast<uint32_t>(h->gw));
  for (const Unit& u : units) {
    int e = 0;
    if (u.ck.h0 == 0) {
      // every head of the unit's states; a state's later head chunks reuse its scratch
      dp.state0 = u.ck.g0;
      e = launch_dequant(h->D, dp, u.ck.n, h->stream);
      if (m + w > 0) h->launches++;
      if (e) return h->cuda_fail(static_cast<cudaError_t>(e));
    }
    if (cudaError_t wt = io_before(u.c)) return h->cuda_fail(wt);
    ap.state0 = u.ck.g0;
    ap.head0 = u.ck.h0;
    ap.nheads = u.ck.nh;
    e = launch_attend(h->D, ap, mq, km, vm, u.ck.n, h->stream);
    h->launches++;
    if (e) return h->cuda_fail(static_cast<cudaError_t>(e));
    if (cudaError_t wt = io_after(u.c)) return h->cuda_fail(wt);
  }
  return CONVKV_OK;
}

int convkv_attend(convkv_t* h, const void* q, void* out) {
  if (!h || (!h->dry && (!q || !out))) return CONVKV_ERR_INVALID_ARG;
  if (h->blocks < 1 || h->need_append || (h->Rs > 0 && !h->sink_set)) return CONVKV_ERR_BAD_ORDER;
  if (h->dry) return CONVKV_OK;
  return attend_impl(h, q, out, nullptr, nullptr);
}

int convkv_attend_sp(convkv_t* h, const void* const* q_shards, void* const* out_shards) {
  if (!h || h->G < 2) return CONVKV_ERR_INVALID_ARG;
  if (!h->dry && !shards_ok(h, q_shards, reinterpret_cast<const void* const*>(out_shards)))
    return CONVKV_ERR_INVALID_ARG;
  if (h->blocks < 1 || h->need_append || (h->Rs > 0 && !h->sink_set)) return CONVKV_ERR_BAD_ORDER;
  if (h->dry) return CONVKV_OK;
  return attend_impl(h, nullptr, nullptr, q_shards, out_shards);
}

// Copies of `bps` bytes per state (blocks of `frames` frames) from host to device
// staging, chunk by chunk on the copy stream, each chunk's completion recorded in its
// event.  A chunk's copy waits only until the previous host-buffer call no longer
// reads that chunk's staging (its kernels of the chunk are done), so it overlaps the
// previous call's later chunks.
static cudaError_t copy_in_chunks(convkv_t* h, void* const* dst, const void* const* src, int nbuf, size_t bps,
                                  int frames) {
  cudaError_t e = cudaSuccess;
  for (int c = 0; c < h->io_nchunks && e == cudaSuccess; ++c) {
    e = cudaStreamWaitEvent(h->io_in, h->ev_done(h->io_prev(c, frames)), 0);
    for (int i = 0; i < nbuf && e == cudaSuccess; ++i)
      e = copy_chunk(h, h->io_chunks[c], dst[i], src[i], bps, cudaMemcpyHostToDevice, h->io_in);
    if (e == cudaSuccess) e = cudaEventRecord(h->ev_in(c), h->io_in);
  }
  return e;
}

// Waits for everything the handle's three streams hold; the first error.
static int sync_all(convkv_t* h) {
  h->io_inflight = false;
  const cudaError_t e1 = cudaStreamSynchronize(h->io_in);
  const cudaError_t e2 = cudaStreamSynchronize(h->io_back);
  const cudaError_t e3 = cudaStreamSynchronize(h->stream);
  if (e1 != cudaSuccess) return h->cuda_fail(e1);
  if (e2 != cudaSuccess) return h->cuda_fail(e2);
  if (e3 != cudaSuccess) return h->cuda_fail(e3);
  return CONVKV_OK;
}

int convkv_append_block_host(convkv_t* h, const void* k_host, const void* v_host, int frames) {
  if (!h || !k_host || !v_host || frames < 1 || frames > h->Bmax) return CONVKV_ERR_INVALID_ARG;
  if (!h->host_io || h->dry) return CONVKV_ERR_BAD_ORDER;
  const size_t bps = static_cast<size_t>(frames) * h->frame_elems() * 2;
  void* const dst[2] = {h->io_k, h->io_v};
  const void* const src[2] = {k_host, v_host};
  h->io_begin(false);
  cudaError_t e = copy_in_chunks(h, dst, src, 2, bps, frames);
  if (e != cudaSuccess) {
    sync_all(h);
    return h->cuda_fail(e);
  }
  // the conv of the evicted frames runs while the block is copied in; the ring append
  // of each chunk waits for that chunk's copy
  h->io_pending = true;
  const int rc = convkv_append_block(h, h->io_k, h->io_v, frames);
  h->io_pending = false;
  h->io_end(frames, false);
  // the caller may reuse its buffers once this returns
  e = cudaStreamSynchronize(h->io_in);
  if (rc != CONVKV_OK) return rc;
  if (e != cudaSuccess) return h->cuda_fail(e);
  return CONVKV_OK;
}

int convkv_attend_host(convkv_t* h, const void* q_host, void* out_host) {
  if (!h || !q_host || !out_host) return CONVKV_ERR_INVALID_ARG;
  if (!h->host_io || h->dry || h->blocks < 1 || h->need_append) return CONVKV_ERR_BAD_ORDER;
  if (h->Rs > 0 && !h->sink_set) return CONVKV_ERR_BAD_ORDER;
  const size_t bps = static_cast<size_t>(h->bcur) * h->frame_elems() * 2;
  void* const dst[1] = {h->io_q};
  const void* const src[1] = {q_host};
  // queries in by chunks; each chunk's attention waits for its queries and its
  // outputs go back on the second copy stream while later chunks compute
  h->io_begin(false);
  cudaError_t e = copy_in_chunks(h, dst, src, 1, bps, h->bcur);
  int rc = CONVKV_OK;
  if (e == cudaSuccess) rc = attend_impl(h, h->io_q, h->io_out, nullptr, nullptr, static_cast<char*>(out_host));
  h->io_end(h->bcur, false);
  const int rs = sync_all(h);
  if (e != cudaSuccess) return h->cuda_fail(e);
  if (rc != CONVKV_OK) return rc;
  return rs;
}

// The enqueue of one host-buffer step (convkv_step_host_async); on failure everything
// already queued is waited for, and the step is undone as a failed append.
static int step_host_enqueue(convkv_t* h, const void* k_host, const void* v_host, const void* q_host,
                             void* out_host, int frames, bool queued) {
  if (!h || !k_host || !v_host || !q_host || !out_host || frames < 1 || frames > h->Bmax)
    return CONVKV_ERR_INVALID_ARG;
  if (!h->host_io || h->dry) return CONVKV_ERR_BAD_ORDER;
  if (h->Rs > 0 && !h->sink_set) return CONVKV_ERR_BAD_ORDER;
  const size_t bps = static_cast<size_t>(frames) * h->frame_elems() * 2;
  void* const dst[3] = {h->io_k, h->io_v, h->io_q};
  const void* const src[3] = {k_host, v_host, q_host};
  h->io_begin(queued);
  cudaError_t e = copy_in_chunks(h, dst, src, 3, bps, frames);
  if (e != cudaSuccess) {
    h->io_end(frames, false);
    sync_all(h);
    return h->cuda_fail(e);
  }
  // bookkeeping, conv, time table and key rotation for all states (while the block is
  // copied in); then per chunk (of states, or of one state's heads): its ring append,
  // its attention, its outputs back -- a chunk's kernels wait only for its own inputs
  const int64_t P = h->P, E = h->E, Sn = h->Sn, blocks = h->blocks;
  const int bcur = h->bcur, last_groups = h->last_groups;
  h->io_pending = true;
  h->io_defer = true;
  int rc = convkv_append_block(h, h->io_k, h->io_v, frames);
  h->io_defer = false;
  for (int c = 0; rc == CONVKV_OK && c < h->io_nchunks; ++c) {
    rc = ring_append_chunk(h, h->io_ap, h->io_k, h->io_v, h->io_chunks[c], c);
    if (rc == CONVKV_OK)
      rc = attend_impl(h, h->io_q, h->io_out, nullptr, nullptr, static_cast<char*>(out_host), c, c + 1);
    if (rc != CONVKV_OK) {
      // as a failed append (later chunks are not appended): counters back, attends
      // refused until an append succeeds, which rewrites the same ring slots
      h->P = P;
      h->E = E;
      h->Sn = Sn;
      h->blocks = blocks;
      h->bcur = bcur;
      h->last_groups = last_groups;
      h->need_append = true;
    }
  }
  h->io_pending = false;
  h->io_end(frames, queued && rc == CONVKV_OK);
  if (rc != CONVKV_OK) sync_all(h);
  return rc;
}

int convkv_step_host_async(convkv_t* h, const void* k_host, const void* v_host, const void* q_host, void* out_host,
                           int frames) {
  return step_host_enqueue(h, k_host, v_host, q_host, out_host, frames, true);
}

int convkv_step_host(convkv_t* h, const void* k_host, const void* v_host, const void* q_host, void* out_host,
                     int frames) {
  const int rc = step_host_enqueue(h, k_host, v_host, q_host, out_host, frames, false);
  if (rc != CONVKV_OK) return rc;
  return sync_all(h);
}

int convkv_sync(convkv_t* h) {
  if (!h) return CONVKV_ERR_INVALID_ARG;
  if (h->dry) return CONVKV_OK;
  if (!h->host_io) {
    const cudaError_t e = cudaStreamSynchronize(h->stream);
    return e == cudaSuccess ? CONVKV_OK : h->cuda_fail(e);
  }
  return sync_all(h);
}

int convkv_host_chunks(const convkv_t* h, int queued, int32_t* rec, int cap) {
  if (!h || (cap > 0 && !rec) || cap < 0) return CONVKV_ERR_INVALID_ARG;
  const std::vector<IoChunk>& plan = h->io_plan[queued ? 1 : 0];
  const int n = static_cast<int>(plan.size());
  for (int c = 0; c < n && c < cap; ++c) {
    const IoChunk& k = plan[c];
    rec[4 * c] = k.g0;
    rec[4 * c + 1] = k.n;
    rec[4 * c + 2] = k.h0;
    rec[4 * c + 3] = k.nh;
  }
  return n;
}

int convkv_layout(const convkv_t* h, int32_t* rec, int cap) {
  if (!h || (cap > 0 && !rec) || cap < 0) return CONVKV_ERR_INVALID_ARG;
  const int r = h->Rs, m = h->m(), w = h->w(), b = h->bcur;
  int n = 0;
  auto put = [&](int part, int64_t src, int64_t phys, int t) {
    if (n < cap) {
      rec[4 * n + 0] = part;
      rec[4 * n + 1] = static_cast<int32_t>(src);
      rec[4 * n + 2] = static_cast<int32_t>(phys);
      rec[4 * n + 3] = t;
    }
    ++n;
  };
  for (int i = 0; i < r; ++i) put(3, i, i, i);
  for (int i = 0; i < m; ++i) {
    const int64_t k = h->Sn - m + i;
    put(0, k, k % h->C, r + i);
  }
  for (int i = 0; i < w; ++i) put(1, h->E + i, (h->E + i) % h->R, r + m + i);
  for (int f = 0; f < b; ++f) put(2, h->P + f, h->fp8 ? f : (h->P + f) % h->R, r + m + w + f);
  return n;
}

int convkv_counters(const convkv_t* h, int64_t out[8]) {
  if (!h || !out) return CONVKV_ERR_INVALID_ARG;
  out[0] = h->P;
  out[1] = h->E;
  out[2] = h->Sn;
  out[3] = h->m();
  out[4] = h->w();
  out[5] = h->bcur;
  out[6] = h->blocks;
  out[7] = h->last_groups;
  return CONVKV_OK;
}

static int read_frame(const convkv_t* hc, const void* dev_base, const uint8_t* bs_base, int nslots, int state,
                      int slot, void* host_dst, const float* scales, int kv, float* host_scales) {
  convkv_t* h = const_cast<convkv_t*>(hc);
  const size_t fe = static_cast<size_t>(h->frame_elems());
  const size_t fb = h->fp4 ? fe / 2 : fe * (h->fp8 ? 1 : 2);
  const char* src = static_cast<const char*>(dev_base) + (static_cast<size_t>(state) * nslots + slot) * fb;
  cudaError_t e = cudaStreamSynchronize(h->stream);
  if (e == cudaSuccess) e = cudaMemcpy(host_dst, src, fb, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && h->fp4)  // NVFP4: the block scales follow the codes
    e = cudaMemcpy(static_cast<char*>(host_dst) + fb, bs_base + (static_cast<size_t>(state) * nslots + slot) * (fe / 16),
                   fe / 16, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && h->fp8 && host_scales)
    e = cudaMemcpy(host_scales, scales + ((static_cast<size_t>(state) * 2 + kv) * nslots + slot) * h->H,
                   sizeof(float) * h->H, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return h->cuda_fail(e);
  return CONVKV_OK;
}

int convkv_read_slot(const convkv_t* h, int state, int kv, int pos, void* host_dst, float* host_scales) {
  if (!h || !host_dst || state < 0 || state >= h->S || (kv != 0 && kv != 1) || pos < 0 || pos >= h->C)
    return CONVKV_ERR_INVALID_ARG;
  if (h->dry) return CONVKV_ERR_BAD_ORDER;
  return read_frame(h, kv ? h->memV : h->memK, kv ? h->memBV : h->memBK, h->C, state, pos, host_dst, h->mem_scale, kv,
                    host_scales);
}

int convkv_read_ring(const convkv_t* h, int state, int kv, int slot, void* host_dst, float* host_scales) {
  if (!h || !host_dst || state < 0 || state >= h->S || (kv != 0 && kv != 1) || slot < 0 || slot >= h->R)
    return CONVKV_ERR_INVALID_ARG;
  if (h->dry) return CONVKV_ERR_BAD_ORDER;
  return read_frame(h, kv ? h->ringV : h->ringK, kv ? h->ringBV : h->ringBK, h->R, state, slot, host_dst,
                    h->ring_scale, kv, host_scales);
}

int convkv_status(convkv_t* h) {
  if (!h) return CONVKV_ERR_INVALID_ARG;
  if (h->dry) return CONVKV_OK;
  int st = 0;
  cudaError_t e = cudaStreamSynchronize(h->stream);
  if (e == cudaSuccess) e = cudaMemcpy(&st, h->status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && st != 0) e = cudaMemsetAsync(h->status, 0, sizeof(int), h->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(h->stream);
  if (e != cudaSuccess) return h->cuda_fail(e);
  return st == kStatusOk ? CONVKV_OK : CONVKV_ERR_DEVICE_TIMEOUT;
}

}  // extern "C"

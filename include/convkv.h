/*
 * convkv.h -- C ABI of the ConvKV Memory attention step for NVIDIA B200 (sm_100a).
 *
 * The method (SoulX-LiveAct):
 *   - blog walk-through (gongshangzheng.github.io/paper-liveact.html), section
 *     "ConvKV Memory": recent KV is kept exact, older KV is compressed by a
 *     lightweight 1D convolution into a fixed-length long-term memory; the
 *     context is [long-term memory | short-term window | current block]; cached
 *     KV is append-only and compression starts with the third block;
 *   - same page, section "Streaming Pipeline": the conv runs once between
 *     blocks, and the KV footprint is the same for any stream length;
 *   - same page, section "Neighbor Forcing": block-wise causal mask (the current
 *     block sees all history and all of itself);
 *   - digi.china.com press article: RoPE Reset re-aligns position encoding;
 *     aiboss88.com summary, ConvKV Memory bullet: 1D conv at a 5:1 ratio, RoPE
 *     position encoding reset;
 *   - model card (hf.xjtesla.cn/Soul-AILab/LiveAct), Command Line Arguments
 *     table, --fp8_kv_cache: KV stored in FP8, dequantised to BF16 on use.
 *
 * One handle holds the KV cache of `num_states` independent layer/denoising-
 * step states that advance in lock step (same block sizes).  Per block the
 * caller makes one convkv_append_block() and then one convkv_attend().
 *
 * Tensor layout of every q, k, v, out buffer (bf16, row-major, contiguous):
 *     [num_states][frames * T][heads][head_dim]
 * where T = grid_h * grid_w tokens per latent frame and token s of a frame sits
 * at spatial position (row, col) = (s / grid_w, s % grid_w).
 *
 * Errors: every call returns 0 (CONVKV_OK) or a negative CONVKV_ERR_* code.
 * A call that fails validation leaves the state unchanged.  Nothing is thrown
 * across the ABI.  A handle is not thread-safe; all its device work is ordered
 * on the stream given at create.
 */
#ifndef CONVKV_H
#define CONVKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CONVKV_OK 0
#define CONVKV_ERR_INVALID_ARG (-1)    /* null pointer, size out of range, bad config */
#define CONVKV_ERR_UNSUPPORTED (-2)    /* valid but not implemented (e.g. evict_frames != 5) */
#define CONVKV_ERR_BAD_ORDER (-3)      /* attend before any append; handle in dry-run mode */
#define CONVKV_ERR_OOM (-4)            /* device allocation failed at create */
#define CONVKV_ERR_CUDA (-5)           /* a CUDA runtime/driver call failed; see convkv_last_cuda_error */
#define CONVKV_ERR_DEVICE_TIMEOUT (-6) /* a kernel gave up waiting on a barrier and returned early */
#define CONVKV_ERR_SCRATCH_LIMIT (-7)  /* request larger than a fixed scratch area (no-allocation entry point) */

#define CONVKV_KV_BF16 0               /* cache stored in bf16 */
#define CONVKV_KV_FP8_E4M3 1           /* window + memory stored e4m3 with per-(head, frame) fp32 scale */
#define CONVKV_KV_NVFP4 2              /* window + memory stored NVFP4: e2m1 pairs, an e4m3 scale per 16
                                          channels, an fp32 scale per (head, frame) (model card, open-source
                                          plan: FP4 for B-series GPUs, read as NVFP4) */

#define CONVKV_COMPRESS_CONV 0         /* 1D conv, kernel 5, stride 5 (the method) */
#define CONVKV_COMPRESS_MEAN 1         /* mean of the 5 evicted frames (--mean_memory option) */

#define CONVKV_FLAG_DRY_RUN 1          /* bookkeeping only: no device memory, no kernel launches */
#define CONVKV_FLAG_HOST_IO 2          /* also allocate device staging for the *_host entry points */

/* Configuration.  All sizes are positive unless stated. */
typedef struct convkv_cfg {
  int heads;               /* H */
  int head_dim;            /* D: 64 or 128 */
  int grid_h, grid_w;      /* tokens per latent frame T = grid_h * grid_w; UNSUPPORTED when the RoPE
                              tables exceed 256 KB or T * max(ring frames, mem_slots) > 2^30 */
  int first_block_frames;  /* b1: frames of the first block */
  int block_frames;        /* b : frames of later blocks; any append may carry 1..max(b1, b) frames */
  int window_frames;       /* W >= 4: past-block frames kept exact */
  int evict_frames;        /* must be 5 (conv kernel = stride = eviction group) */
  int mem_slots;           /* C >= 1: FIFO capacity of compressed slots */
  int rope_t, rope_h, rope_w; /* RoPE channels per axis (even, sum = D); all 0 -> D-4*floor(D/6), 2*floor(D/6), 2*floor(D/6) */
  double rope_theta;       /* RoPE base, e.g. 1e4 */
  int kv_format;           /* CONVKV_KV_BF16, CONVKV_KV_FP8_E4M3 or CONVKV_KV_NVFP4 */
  int compress_mode;       /* CONVKV_COMPRESS_CONV or CONVKV_COMPRESS_MEAN */
  int num_states;          /* independent states advanced together (>= 1) */
  int flags;               /* CONVKV_FLAG_* */
  int t_offset;            /* added to every RoPE time index (outputs must not depend on it); normally 0 */
  const void* conv_weight; /* device bf16 [num_states][2 (K,V)][H][D_out][D_in][5]; read once at create,
                              not retained; may be NULL for CONVKV_COMPRESS_MEAN or dry-run */
  void* stream;            /* cudaStream_t for all device work of this handle (NULL = legacy default) */
  int sink_frames;         /* reference-image frames attended first and never evicted (0 = none);
                              their K/V are given once with convkv_set_sink */
  int sp_ranks;            /* sequence-parallel group size G, 1..8 (0 or 1: no sharding); with G > 1
                              `heads` is this rank's share of the G*heads heads */
  int sp_rank;             /* this handle's rank g in [0, G): it owns heads [g*heads, (g+1)*heads) */
} convkv_cfg;

typedef struct convkv convkv_t;

/* Validate cfg, allocate the whole device state in one arena (zero-filled),
 * build the RoPE tables, and permute the conv weights into the kernel layout.
 * No device memory is allocated after this call.  *out receives the handle.
 * Errors: INVALID_ARG, UNSUPPORTED, OOM, CUDA. */
int convkv_create(const convkv_cfg* cfg, convkv_t** out);

/* Append one block (SoulX-LiveAct blog, "ConvKV Memory" / "Streaming Pipeline"):
 *   1. the previous current block joins the window;
 *   2. while the window holds more than W frames, its oldest 5 frames are
 *      compressed into one memory slot (FIFO of C slots, oldest dropped);
 *   3. k, v become the current block (copied into the ring; e4m3 + scale in the
 *      fp8 format, with a bf16 copy kept for this block's attend).
 * k, v: DEVICE pointers, [num_states][frames*T][H][D] bf16; the copy is
 * asynchronous on the handle's stream, so keep them unchanged until it passes.
 * frames: 1 .. max(b1, b).  Errors: INVALID_ARG, BAD_ORDER (dry-run with
 * non-null pointers is fine), CUDA.
 * A CUDA error leaves the counters (and so the layout) as they were before the
 * call; a compression that already ran for the call may have rewritten one
 * memory position, so attends return BAD_ORDER until an append succeeds, and
 * that append recomputes the position from the same ring frames. */
int convkv_append_block(convkv_t* h, const void* k, const void* v, int frames);

/* Attention of the current block's queries over [memory | window | current]
 * (preceded by the reference frames when cfg.sink_frames > 0) with RoPE time
 * indices reset to start at 0 (memory slot i -> r + i, window frame j -> r + m +
 * j, current frame f -> r + m + w + f, r = sink_frames), spatial indices
 * unchanged, softmax scale 1/sqrt(D), no mask inside the attended set.
 * BAD_ORDER also when sink_frames > 0 and convkv_set_sink was not called, and
 * after an append that failed, until an append succeeds.
 * q, out: DEVICE pointers, [num_states][frames*T][H][D] bf16 with `frames` of
 * the last append.  Does not change the state (may be repeated).
 * Errors: INVALID_ARG, BAD_ORDER, CUDA. */
int convkv_attend(convkv_t* h, const void* q, void* out);

/* Same as append_block / attend but with HOST buffers (pinned or pageable): the
 * inputs are copied into handle-owned device staging by chunks of states on the
 * handle's own copy stream, and each chunk's ring append or attention starts as soon
 * as that chunk has landed; attend_host copies each chunk's outputs back on a second
 * copy stream while later chunks compute (chunks: one state, then sizes growing 1.3
 * times per chunk up to a steady size of at most 6 states, chosen so that the
 * attention grid of a chunk fills its last wave of SMs best, at most the attention's
 * group of states in the e4m3 / NVFP4 formats; the last chunks shrink to one state.
 * A handle of one state is chunked by ranges of heads instead: see
 * convkv_host_chunks).  Both calls return
 * once the host buffers are no longer accessed: the inputs copied in, the outputs
 * copied back.  With pinned buffers the copies overlap the kernels.  Needs
 * CONVKV_FLAG_HOST_IO at create (which also creates the two copy streams and their
 * events).  Errors: as above, plus BAD_ORDER without the flag. */
int convkv_append_block_host(convkv_t* h, const void* k_host, const void* v_host, int frames);
int convkv_attend_host(convkv_t* h, const void* q_host, void* out_host);

/* One step from and to HOST buffers: append_block_host(k_host, v_host, frames)
 * followed by attend_host(q_host, out_host), with the queries of the new block
 * (`frames` frames).  The inputs are copied in by chunks of states; each chunk's
 * ring append and attention start as soon as its k, v and q have landed, and its
 * outputs go back while later chunks compute (the conv of the evicted frames, the
 * time table and the key rotation run for all states first, while the block is
 * copied in).  Same results, bit for bit, as the two calls.  Returns once the host
 * buffers are no longer accessed.  A failure after the bookkeeping counts as a
 * failed append (counters restored, attends BAD_ORDER until an append succeeds).
 * Needs CONVKV_FLAG_HOST_IO.  Errors: as append_block and attend, plus BAD_ORDER
 * without the flag. */
int convkv_step_host(convkv_t* h, const void* k_host, const void* v_host, const void* q_host, void* out_host,
                     int frames);

/* The same step, returned as soon as it is queued: the copies in of the next step's
 * chunks then overlap this step's later kernels (a chunk's staging is refilled as soon
 * as the previous step's kernels and copy back of that chunk are done), so a stream
 * of steps runs at the rate of the slower of the kernels and the copies.  The host
 * buffers of every queued step must stay valid, the inputs unchanged and the outputs
 * unread, until convkv_sync returns.  Argument and order errors are returned at once
 * with nothing queued; a failure while queueing is waited out and counts as a failed
 * append, as for convkv_step_host; device-side errors show in convkv_sync.  Needs
 * CONVKV_FLAG_HOST_IO. */
int convkv_step_host_async(convkv_t* h, const void* k_host, const void* v_host, const void* q_host,
                           void* out_host, int frames);

/* Waits until every queued call of the handle has ended (its kernels, and with
 * CONVKV_FLAG_HOST_IO its copies in both directions).  Errors: INVALID_ARG, CUDA. */
int convkv_sync(convkv_t* h);

/* Device bytes owned by the handle; constant from create to destroy. */
size_t convkv_state_bytes(const convkv_t* h);

/* Release everything the handle owns (waits for its stream).  NULL is a no-op. */
void convkv_destroy(convkv_t* h);

/* Reference-image partition (SoulX-LiveAct blog, "ConvKV Memory": the KV context
 * is reference-image state + long-term memory + short-term memory + current
 * block).  Stores the K/V of the cfg.sink_frames reference frames: DEVICE
 * pointers, [num_states][sink_frames*T][H][D] bf16, copied asynchronously on
 * the handle's stream (kept in bf16 in both formats).  They are never evicted
 * or compressed and every attend takes them first, so the RoPE time indices run
 * 0.. over [reference | memory | window | current].  May be called again to
 * replace them.  Errors: INVALID_ARG, BAD_ORDER (sink_frames == 0), CUDA. */
int convkv_set_sink(convkv_t* h, const void* k, const void* v);

/* Sequence-parallel forms of append and attend (SoulX-LiveAct blog walk-through,
 * system-level optimisation section, item (2): the sequence dimension is split over
 * two GPUs that synchronise by communication; read here as the all-to-all between
 * sequence shards and head shards, heads being independent in this step).  The caller's activations
 * are split by sequence: rank r holds rows [off_r, off_{r+1}) of the block's
 * frames*T rows, off_r = floor(r * frames*T / G), with ALL G*heads heads, as
 * [num_states][off_{r+1}-off_r][G*heads][D] bf16.  The exchange is fused into the
 * kernels: append gathers this rank's heads of every row from the G shards, attend
 * reads its heads' query rows from the G q shards and writes each output row back
 * into the shard of the rank that holds it.  shards[r] are DEVICE pointers valid in
 * this process (a peer GPU's buffer mapped here, or a local buffer); the arrays
 * themselves are host arrays of cfg.sp_ranks pointers, read during the call.  The
 * caller orders the ranks around each call: every shard is written before any
 * rank's kernels read it, and outputs are read after every rank's attend ends.
 * Errors: as the plain forms; INVALID_ARG when the handle has sp_ranks < 2 or a
 * shard pointer is null. */
int convkv_append_block_sp(convkv_t* h, const void* const* k_shards, const void* const* v_shards, int frames);
int convkv_attend_sp(convkv_t* h, const void* const* q_shards, void* const* out_shards);

/* CUDA IPC helpers for sequence-parallel shards on a multi-GPU node (no counterpart
 * on the pages; plumbing for the fused exchange above).  export: the 64-byte IPC
 * handle of the cudaMalloc allocation that holds dev_ptr, and dev_ptr's byte
 * offset in it (the allocation must come from cudaMalloc, not a virtual-memory
 * pool).  open: maps a handle exported by another process on this node, with peer
 * access enabled on first use; the shard is at *dev_ptr + offset.  close: unmaps
 * a pointer returned by open.  Errors: INVALID_ARG (null argument, pointer not in
 * a device allocation), CUDA. */
int convkv_ipc_export(const void* dev_ptr, void* handle64, size_t* offset);
int convkv_ipc_open(const void* handle64, void** dev_ptr);
int convkv_ipc_close(void* dev_ptr);

/* Key-frame layout of the next attend, in attended order, 4 int32 per frame:
 * {partition (0 memory, 1 window, 2 current, 3 reference image), source index
 * (slot index for memory -- slot k covers stream frames [5k, 5k+5) -- frame
 * index within the reference for the reference image, else stream frame
 * index), physical slot (memory position, ring slot, staging slot for the fp8
 * current block, or reference frame), RoPE time index}.  Returns the number of
 * key frames, or a negative error; writes at most `cap` records. */
int convkv_layout(const convkv_t* h, int32_t* rec, int cap);

/* Chunk plan of the host-buffer entry points, in stream order, 4 int32 per chunk:
 * {first state, states, first head, heads}.  With several states the chunks are
 * whole states (all heads); with one state they are ranges of its heads (strided
 * copies of nh * D values per token).  queued = 0: the plan of a call that follows a
 * synchronised one (it ramps up from one state and down to one); queued != 0: the
 * plan of a queued step (convkv_step_host_async) that follows a queued step (steady
 * chunks; its copies in ran during the previous step).  A handle created with
 * CONVKV_FLAG_HOST_IO has the plans (a dry-run handle too, planned for 148 SMs); any
 * other handle has none.  Returns the number of chunks, or a negative error; writes
 * at most `cap` records. */
int convkv_host_chunks(const convkv_t* h, int queued, int32_t* rec, int cap);

/* Counters {P promoted frames, E evicted frames, S slots produced, m stored
 * slots, w window frames, b current frames, blocks appended, groups compressed
 * by the last append}.  Returns 0 or INVALID_ARG. */
int convkv_counters(const convkv_t* h, int64_t out[8]);

/* Copy one stored memory slot (memory position `pos` in [0, C)) of one state
 * and one of K (kv = 0) or V (kv = 1) to host memory: [T][H][D] bf16, or e4m3
 * bytes in the fp8 format, or in the NVFP4 format [T][H][D/2] bytes of e2m1 pairs
 * (even channel in the low nibble) followed by [T][H][D/16] e4m3 block scales;
 * the fp32 scales[H] of the low-precision formats go to host_scales (may be
 * NULL).  Synchronises the stream.  Errors: INVALID_ARG, BAD_ORDER, CUDA. */
int convkv_read_slot(const convkv_t* h, int state, int kv, int pos, void* host_dst, float* host_scales);

/* Copy one ring frame slot (`slot` in [0, W + max(b1, b))) the same way. */
int convkv_read_ring(const convkv_t* h, int state, int kv, int slot, void* host_dst, float* host_scales);

/* Synchronise the stream, return CONVKV_OK or the first error recorded by a
 * kernel (DEVICE_TIMEOUT), and clear the device status word. */
int convkv_status(convkv_t* h);

/* Number of kernels this handle has launched so far. */
int64_t convkv_launch_count(const convkv_t* h);

/* Self-test of the bounded device waits (failure detection): launches one CTA
 * that waits on a barrier nothing arrives on, with a budget of budget_clocks SM
 * clocks (1000 .. 2e9).  The wait gives up, the kernel writes the timeout code
 * to *dev_status (DEVICE int, caller-owned, zero on entry) and returns; the
 * call synchronises `stream` and returns CONVKV_ERR_DEVICE_TIMEOUT -- the
 * expected result -- or CONVKV_OK if the wait somehow completed.  The context
 * stays usable.  Errors: INVALID_ARG, CUDA. */
int convkv_selftest_wait_timeout(int* dev_status, long long budget_clocks, void* stream);

/* Self-test of the quantisers' division (the e4m3 / NVFP4 codes are decided by
 * fp32 quotients x / scale rounded to nearest, as the FP8 / FP4 cache formats of
 * the SoulX-LiveAct model card store them): for each of the n pairs
 * (dev_x[i], dev_s[i]) (DEVICE fp32 arrays, caller-owned) the kernels' shared-
 * divisor quotient is compared bit for bit with CUDA's IEEE division, and the
 * number of differing pairs is added to *dev_mismatches (DEVICE unsigned int,
 * caller-owned).  Synchronises `stream`.  Errors: INVALID_ARG, CUDA. */
int convkv_selftest_div_rn(const float* dev_x, const float* dev_s, int64_t n, unsigned int* dev_mismatches,
                           void* stream);

/* Failure injection for tests, on the host: the `step`-th launch step (0-based,
 * counted per call: conv, time-table upload, ring append; in dry-run handles the
 * steps are counted but not run) of the next append reports cudaErrorLaunchFailure
 * instead of running, once; -1 disarms.  Errors: INVALID_ARG. */
int convkv_debug_fail_step(convkv_t* h, int step);

/* cudaError_t of the last failing CUDA call made through this handle (0 if none). */
int convkv_last_cuda_error(const convkv_t* h);

/* Static description of an error code. */
const char* convkv_strerror(int code);

/* ------------------------------------------------------------------------
 * Allocation-free quantiser.  The paper has no counterpart of this call; it
 * exists for callers that cannot allocate device memory while they run -- a
 * serving engine that hands out every device byte from its own fixed pool, or
 * a thread on a latency-critical path where cudaMalloc would synchronise the
 * device and stall its other streams.
 *
 * Quantises `frames` bf16 frames x [frames][tokens][heads][head_dim] (DEVICE)
 * to e4m3 exactly as the fp8 append does (per frame and head: scale =
 * amax / 448, 1 if amax is 0; code = e4m3(x / scale), IEEE fp32 divide,
 * round-to-nearest-even, saturating to +-448) and writes the codes to `codes`
 * (DEVICE, same layout, 1 byte each) and the scales to `scales` (DEVICE fp32
 * [frames][heads]), asynchronously on `stream` (cudaStream_t, NULL = legacy
 * default).  The caller owns all three buffers.
 *
 * Alignment: x on 16 bytes, codes on 8, scales on 4 (a misaligned pointer
 * returns INVALID_ARG before anything runs).
 *
 * No device memory is allocated by a call: the only scratch, one amax per
 * (frame, head), is a fixed array of CONVKV_NOALLOC_MAX_FRAME_HEADS entries
 * (16 KiB) inside the library, kept on every GPU that loads the library until
 * the process exits.  frames * heads above that limit returns
 * CONVKV_ERR_SCRATCH_LIMIT.  The first call on a device resolves the array's
 * address there (with that device current); with lazy module loading that
 * first call may also make the driver load this part of the library's device
 * code, the array included.  So make the first call once during set-up, before
 * any stream capture and outside any window in which allocation is forbidden.
 * The resolved address is kept for the life of the process: calling
 * cudaDeviceReset on a device after its first call is not supported.  Every
 * call shares the array and it keeps the last call's contents (each call
 * clears the part it uses), so calls whose work overlaps on the GPU -- on
 * different streams, or from several host threads at once -- race and give
 * wrong results.  head_dim must be a multiple of 8.  Errors: INVALID_ARG,
 * SCRATCH_LIMIT, UNSUPPORTED (device ordinal >= 128), CUDA. */
#define CONVKV_NOALLOC_MAX_FRAME_HEADS 4096
int convkv_quantize_e4m3_noalloc(const void* x, void* codes, float* scales, int frames, int tokens, int heads,
                                 int head_dim, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CONVKV_H */

"""fp64 CPU oracle for the ConvKV Memory attention step.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path (the
C-ABI library and its Python binding) never calls it and has no CPU fallback.
It shares no code with the CUDA path; the only common dependency is the seeded
input generator, which holds none of the method's arithmetic.

What it computes, and where that is stated:

* SoulX-LiveAct blog walk-through (gongshangzheng.github.io/paper-liveact.html),
  section "ConvKV Memory": recent KV is kept exact, older KV is compressed by a
  lightweight 1D convolution into a fixed-length long-term memory; the context
  is [long-term memory | short-term memory | current block]; cached KV is
  append-only; compression starts with the third generated block.
* Same page, section "Streaming Pipeline": the conv runs once between blocks,
  and the KV footprint is constant for any stream length.
* Same page, section "Neighbor Forcing": block-wise causal mask -- the current
  block sees all history and all of itself (no mask inside the attended set).
* digi.china.com press article (third technical paragraph): old KV is rolled
  into a fixed-length representation at a fixed compression ratio, and RoPE
  Reset re-aligns the position encoding.
* aiboss88.com summary, section "SoulX-LiveActの技術的原理", ConvKV Memory
  bullet: the 1D convolution compresses at 5:1 and the RoPE position encoding
  is reset.
* Model card (hf.xjtesla.cn/Soul-AILab/LiveAct), "Command Line Arguments"
  table, ``--fp8_kv_cache``: the KV cache is stored in FP8 and dequantised to
  BF16 on use.
* Same model card, open-source plan: FP4 for B-series GPUs (planned, format not
  given).  Read as NVFP4, the Blackwell 4-bit format: e2m1 values with one e4m3
  scale per 16 consecutive channels and one fp32 scale per (frame, head), stored
  and dequantised to BF16 on use like the FP8 cache.

Readings taken where the pages are silent (each listed in the design notes):
W counts past-block frames only and eviction happens at append time in
groups of 5 until the window holds at most W frames; the memory is a FIFO of
C slots (oldest dropped); the conv is a per-head cross-correlation over the 5
evicted frames (tap j = j-th oldest frame), no bias, applied to un-rotated K
and V; compressed slots are stored in the cache's storage type (bf16 rounded
to nearest even, or e4m3 with a per-(head, slot) fp32 scale); an e4m3 value is
dequantised to BF16 on use as bf16(fp32(code * scale)), so every consumer (the
conv of evicted window frames, the attention over window and memory) reads
that bf16 value; RoPE time
indices restart at 0 over [memory | window | current], one index per memory
slot, spatial (row, column) indices are kept; RoPE rotates adjacent pairs of
each axis segment [t | h | w] with frequency theta^(-2i/d_axis); softmax scale
is 1/sqrt(D).  In the fp8 variant the current block is attended in bf16 and is
quantised when it joins the window.

Parity status: every function below is pinned by tests under ``tests/`` that
check it against closed forms, library routines or hand-derived tables (no
function is left unpinned).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import numpy as np

# Partition codes of a key frame in the attended sequence.
PART_MEMORY, PART_WINDOW, PART_CURRENT, PART_SINK = 0, 1, 2, 3
EVICT = 5          # frames per eviction group = conv kernel = conv stride (5:1)
E4M3_MAX = 448.0   # largest finite e4m3 value
E2M1_MAX = 6.0     # largest finite e2m1 value
FP4_BLOCK = 16     # channels per NVFP4 block scale


# --------------------------------------------------------------------------
# bf16 / e4m3 storage rounding
# --------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even).

    The cache stores K/V in bf16; a compressed slot is stored in the same type.
    Done on the exact binary expansion: bf16 keeps 8 significant bits, so the
    value is rounded at the bit below the 8th significant bit.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    m, e = np.frexp(x[nz])              # x = m * 2^e, 0.5 <= |m| < 1
    q = np.round(m * 256.0)              # 8 significant bits, numpy rounds half to even
    out[nz] = np.ldexp(q / 256.0, e)
    return out


def e4m3_rne_satfinite(x32: np.ndarray) -> np.ndarray:
    """fp32 -> nearest e4m3 value (ties to even), saturating to +-448.

    e4m3 (OCP FP8): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; normal
    numbers 2^-6 .. 448, subnormals are multiples of 2^-9.  A value with
    exponent e (|x| in [2^e, 2^(e+1))) has quantum 2^(e-3); below 2^-6 the
    quantum is 2^-9.  Values beyond 448 saturate to 448.
    """
    x = np.asarray(x32, dtype=np.float32).astype(np.float64)
    a = np.abs(x)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))   # a = m * 2^ex, 0.5 <= m < 1
    e = np.maximum(ex.astype(np.float64) - 1.0, -6.0)
    quantum = np.exp2(e - 3.0)
    q = np.round(a / quantum) * quantum   # exact: a and quantum are dyadic
    q = np.minimum(q, E4M3_MAX)
    return np.where(a > 0, np.copysign(q, x), 0.0 * x)


def fp8_encode(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per-head e4m3 codes of one frame or slot x[T, H, D].

    scale = amax / 448 in fp32 (1 if amax == 0); code = e4m3(fp32(x) / scale)
    with the fp32 divide rounded to nearest.  Returns (code values as float64,
    scales[H] as float32).
    """
    x = np.asarray(x, dtype=np.float64)
    x32 = x.astype(np.float32)
    amax = np.abs(x32).max(axis=(0, 2))                      # [H], fp32
    scale = np.where(amax == 0, np.float32(1.0), (amax / np.float32(E4M3_MAX)).astype(np.float32))
    scale = scale.astype(np.float32)
    y = (x32 / scale[None, :, None]).astype(np.float32)      # IEEE fp32 divide
    return e4m3_rne_satfinite(y), scale


def fp8_dequantize(code: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """Dequantise to BF16 on use: bf16(fp32(code * scale)), scale per head (axis 1)."""
    prod = (np.asarray(code, dtype=np.float32) * np.asarray(scale, dtype=np.float32)[None, :, None]).astype(np.float32)
    return round_to_bf16(prod.astype(np.float64))


def fp8_quantize(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """e4m3 storage of x[T, H, D] followed by the bf16 dequantisation used by every
    consumer (conv input, attention K/V).  Returns (dequantised values, scales[H])."""
    code, scale = fp8_encode(x)
    return fp8_dequantize(code, scale), scale


def e2m1_rne_satfinite(x32: np.ndarray) -> np.ndarray:
    """fp32 -> nearest e2m1 value (ties to even), saturating to +-6.

    e2m1 (OCP FP4): 1 sign, 2 exponent bits (bias 1), 1 mantissa bit; the
    magnitudes are 0, 0.5 (subnormal), 1, 1.5, 2, 3, 4, 6.  A value with exponent
    e >= 0 (|x| in [2^e, 2^(e+1))) has quantum 2^(e-1); below 1 the quantum is
    1/2.  Ties go to the even multiple of the quantum (mantissa bit 0).
    """
    x = np.asarray(x32, dtype=np.float32).astype(np.float64)
    a = np.abs(x)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))   # a = m * 2^ex, 0.5 <= m < 1
    e = np.maximum(ex.astype(np.float64) - 1.0, 0.0)
    quantum = np.exp2(e - 1.0)
    q = np.round(a / quantum) * quantum          # exact: a and quantum are dyadic
    q = np.minimum(q, E2M1_MAX)
    return np.where(a > 0, np.copysign(q, x), 0.0 * x)


def fp4_encode(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """NVFP4 codes of one frame or slot x[T, H, D], in fp32 steps:

      g   = amax / (448 * 6) per head over the frame's [T, D] (1 if amax == 0)
      s_b = e4m3(a_b / (g * 6)) per block b of 16 channels of a token, a_b = max|x| in b
      e_b = s_b * g
      code = e2m1(x / e_b)   (0 where e_b == 0)

    every product and quotient rounded to nearest in fp32, e4m3 and e2m1 rounding
    to nearest even with saturation.  Returns (code values [T, H, D], block scale
    values [T, H, D/16] (e4m3, as float64), tensor scales [H] (float32)).
    """
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    T, H, D = x32.shape
    amax = np.abs(x32).max(axis=(0, 2))
    g = np.where(amax == 0, np.float32(1.0),
                 (amax / np.float32(E4M3_MAX * E2M1_MAX)).astype(np.float32)).astype(np.float32)
    xb = x32.reshape(T, H, D // FP4_BLOCK, FP4_BLOCK)
    ab = np.abs(xb).max(axis=3)                                          # [T, H, nb], fp32
    denom = (g * np.float32(E2M1_MAX)).astype(np.float32)                # [H]
    ratio = (ab / denom[None, :, None]).astype(np.float32)
    sb = e4m3_rne_satfinite(ratio)                                       # e4m3 values
    eb = (sb.astype(np.float32) * g[None, :, None]).astype(np.float32)   # effective scale
    safe = np.where(eb > 0, eb, np.float32(1.0)).astype(np.float32)
    y = (xb / safe[..., None]).astype(np.float32)
    code = np.where(eb[..., None] > 0, e2m1_rne_satfinite(y), 0.0)
    return code.reshape(T, H, D), sb, g


def fp4_dequantize(code: np.ndarray, sb: np.ndarray, g: np.ndarray) -> np.ndarray:
    """Dequantise to BF16 on use: bf16(fp32(code * fp32(s_b * g)))."""
    T, H, D = code.shape
    eb = (np.asarray(sb, dtype=np.float32) * np.asarray(g, dtype=np.float32)[None, :, None]).astype(np.float32)
    c = np.asarray(code, dtype=np.float32).reshape(T, H, D // FP4_BLOCK, FP4_BLOCK)
    prod = (c * eb[..., None]).astype(np.float32)
    return round_to_bf16(prod.astype(np.float64)).reshape(T, H, D)


# --------------------------------------------------------------------------
# RoPE with reset positions
# --------------------------------------------------------------------------

def rope_split(D: int) -> Tuple[int, int, int]:
    """Channel split (time, row, column) of head_dim D: 44/42/42 for D=128.

    Row and column each get 2*floor(D/6) channels, time gets the rest.
    """
    dh = 2 * (D // 6)
    return D - 2 * dh, dh, dh


def rope_angles(t: np.ndarray, y: np.ndarray, xc: np.ndarray, split: Tuple[int, int, int],
                theta: float) -> np.ndarray:
    """Rotation angle of every channel pair at positions (t, y, xc): [..., D/2].

    Pairs [0, d_t/2) follow the time index, the next d_h/2 the row index, the
    rest the column index; pair i of an axis segment of width d turns by
    pos * theta^(-2i/d).
    """
    parts = []
    for width, pos in zip(split, (t, y, xc)):
        i = np.arange(width // 2, dtype=np.float64)
        freq = theta ** (-2.0 * i / width)
        parts.append(np.asarray(pos, dtype=np.float64)[..., None] * freq)
    shape = np.broadcast_shapes(*[p.shape[:-1] for p in parts])
    return np.concatenate([np.broadcast_to(p, shape + p.shape[-1:]) for p in parts], axis=-1)


def rope_apply(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Turn each adjacent channel pair (2i, 2i+1) of x[..., D] by the angle whose
    cosine and sine are cos[..., i], sin[..., i]: (a, b) -> (a cos - b sin, a sin + b cos)."""
    x = np.asarray(x, dtype=np.float64)
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, cos.shape[:-1] + (x.shape[-1],)))
    out[..., 0::2] = a * cos - b * sin
    out[..., 1::2] = a * sin + b * cos
    return out


def rope_rotate(x: np.ndarray, t: np.ndarray, y: np.ndarray, xc: np.ndarray,
                split: Tuple[int, int, int], theta: float) -> np.ndarray:
    """Rotate x[..., D] by 3D RoPE at positions (t, y, xc) (broadcast over x[..., 0]).

    Channels [0, d_t) use the time index, [d_t, d_t+d_h) the row index and the
    rest the column index.  Inside an axis segment of width d, pair i (channels
    2i, 2i+1 of the segment) turns by angle pos * theta^(-2i/d).
    """
    ang = rope_angles(t, y, xc, split, theta)
    return rope_apply(x, np.cos(ang), np.sin(ang))


# --------------------------------------------------------------------------
# 1D conv compression of one eviction group
# --------------------------------------------------------------------------

def conv_compress(group: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Compress 5 frames group[5, T, H, D] into one slot [T, H, D].

    out[s, h, o] = sum_j sum_i w[h, o, i, j] * group[j, s, h, i]
    (per-head channel mixing, kernel 5 = stride 5 over time, no padding,
    no bias, tap j = j-th oldest frame).  Per head this is one matrix product
    over the combined (j, i) index: [T x 5D] . [5D x D].
    """
    g = np.asarray(group, dtype=np.float64)
    wf = np.asarray(w, dtype=np.float64)
    assert g.shape[0] == EVICT and wf.shape[-1] == EVICT
    n, T, H, D = g.shape
    out = np.empty((T, H, wf.shape[1]))
    for h in range(H):
        x = g[:, :, h, :].transpose(1, 0, 2).reshape(T, EVICT * D)      # [s, (j, i)]
        wt = wf[h].transpose(2, 1, 0).reshape(EVICT * D, wf.shape[1])   # [(j, i), o]
        out[:, h, :] = x @ wt
    return out


# --------------------------------------------------------------------------
# attention of query rows over one key/value sequence
# --------------------------------------------------------------------------

def attend_rows(q_rot: np.ndarray, k_rot: np.ndarray, v: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """softmax(q k^T / sqrt(D)) v for one head, unmasked.

    q_rot[n, D], k_rot[Nk, D], v[Nk, D] -> (o[n, D], sum of the normalised
    weights per row, which is 1 up to rounding).
    """
    D = q_rot.shape[-1]
    s = (q_rot @ k_rot.T) / np.sqrt(D)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    l = p.sum(axis=1, keepdims=True)
    p = p / l
    return p @ v, p.sum(axis=1)


# --------------------------------------------------------------------------
# the streaming state of one layer / denoising step
# --------------------------------------------------------------------------

@dataclass
class OracleConfig:
    H: int
    D: int
    grid_h: int
    grid_w: int
    window: int            # W, past-block frames kept exact
    mem_slots: int         # C, FIFO capacity of compressed slots
    theta: float = 1e4
    fp8: bool = False
    fp4: bool = False      # NVFP4 storage (exclusive with fp8)
    split: Optional[Tuple[int, int, int]] = None

    @property
    def T(self) -> int:
        return self.grid_h * self.grid_w

    def rope(self) -> Tuple[int, int, int]:
        return self.split if self.split is not None else rope_split(self.D)


@dataclass
class _Frame:
    k: np.ndarray          # [T, H, D] float64 (stored values, as consumed)
    v: np.ndarray
    index: int             # stream frame index (window/current) or slot index (memory)
    codes: Optional[tuple] = None   # fp8: (k codes, k scales, v codes, v scales);
                                    # fp4: scales are (block scales, tensor scales)


@dataclass
class ConvEvent:
    block: int             # 1-based block number of the append that ran it
    first_frame: int       # stream index of the oldest evicted frame (g0)
    slot: int              # slot index S-1 (covers frames [5*slot, 5*slot+5))


class OracleStream:
    """Reference state machine for one layer / denoising-step KV cache."""

    def __init__(self, cfg: OracleConfig, conv_w: np.ndarray):
        """conv_w: [2 (K, V), H, D_out, D_in, 5], float64 (exact bf16 values)."""
        self.cfg = cfg
        self.w = np.asarray(conv_w, dtype=np.float64)
        self.window: List[_Frame] = []
        self.current: List[_Frame] = []
        self.current_q8: List[_Frame] = []   # fp8: quantised form of the current frames
        self.memory: List[_Frame] = []
        self.P = 0        # frames promoted into the window so far
        self.E = 0        # frames evicted so far
        self.S = 0        # slots produced so far
        self.block = 0
        self.events: List[ConvEvent] = []
        self.mem_scales: List[tuple] = []       # fp8/fp4: per-slot (K, V) scales
        self.frame_scales = {}                  # fp8/fp4: stream frame -> (K, V) scales
        self.sink: List[_Frame] = []            # reference-image frames, never evicted

    # -- reference-image partition -------------------------------------------
    def set_sink(self, k: np.ndarray, v: np.ndarray) -> None:
        """Reference-image state (SoulX-LiveAct blog, "ConvKV Memory": the context is
        reference-image state + long-term memory + short-term memory + current block).
        k, v[n, T, H, D]: kept exact, never evicted or compressed, attended first."""
        self.sink = [_Frame(np.asarray(k[i], dtype=np.float64), np.asarray(v[i], dtype=np.float64), i)
                     for i in range(k.shape[0])]

    # -- append ------------------------------------------------------------
    def append(self, k: np.ndarray, v: np.ndarray) -> List[ConvEvent]:
        """Append one block k, v[b, T, H, D] (exact input values)."""
        cfg = self.cfg
        self.block += 1
        # (i) the previous current block joins the window
        promoted = self.current_q8 if (cfg.fp8 or cfg.fp4) else self.current
        self.window.extend(promoted)
        self.P += len(promoted)
        self.current, self.current_q8 = [], []
        # (ii) evict the oldest 5 frames while the window holds more than W
        new_events = []
        while len(self.window) > cfg.window:
            group, self.window = self.window[:EVICT], self.window[EVICT:]
            kc = conv_compress(np.stack([f.k for f in group]), self.w[0])
            vc = conv_compress(np.stack([f.v for f in group]), self.w[1])
            codes = None
            if cfg.fp8 or cfg.fp4:
                (kc, ck, sk), (vc, cv, sv) = self._quantize(kc), self._quantize(vc)
                scales = (sk, sv)
                codes = (ck, sk, cv, sv)
            else:
                kc, vc = round_to_bf16(kc), round_to_bf16(vc)
                scales = None
            if len(self.memory) == cfg.mem_slots:
                self.memory.pop(0)
                self.mem_scales.pop(0)
            self.memory.append(_Frame(kc, vc, self.S, codes))
            self.mem_scales.append(scales)
            ev = ConvEvent(self.block, group[0].index, self.S)
            self.E += EVICT
            self.S += 1
            self.events.append(ev)
            new_events.append(ev)
        # (iii) the new block becomes the current block
        b = k.shape[0]
        for f in range(b):
            idx = self.P + f
            kf = np.asarray(k[f], dtype=np.float64)
            vf = np.asarray(v[f], dtype=np.float64)
            self.current.append(_Frame(kf, vf, idx))
            if cfg.fp8 or cfg.fp4:
                (kq, ck, sk), (vq, cv, sv) = self._quantize(kf), self._quantize(vf)
                self.current_q8.append(_Frame(kq, vq, idx, (ck, sk, cv, sv)))
                self.frame_scales[idx] = (sk, sv)
        return new_events

    def _quantize(self, x: np.ndarray):
        """(values as consumed, codes, scales) of one frame or slot in the cache's
        low-precision format; fp4 scales are (block scales, tensor scales)."""
        if self.cfg.fp4:
            code, sb, g = fp4_encode(x)
            return fp4_dequantize(code, sb, g), code, (sb, g)
        code, scale = fp8_encode(x)
        return fp8_dequantize(code, scale), code, scale

    # -- layout ------------------------------------------------------------
    def key_frames(self) -> List[Tuple[int, _Frame, int]]:
        """(partition, frame, RoPE time index) in attended order:
        [reference image | memory | window | current], time indices from 0."""
        out = []
        t = 0
        for f in self.sink:
            out.append((PART_SINK, f, t)); t += 1
        for f in self.memory:
            out.append((PART_MEMORY, f, t)); t += 1
        for f in self.window:
            out.append((PART_WINDOW, f, t)); t += 1
        for f in self.current:
            out.append((PART_CURRENT, f, t)); t += 1
        return out

    def layout(self) -> np.ndarray:
        """int64 rows (partition, source index, RoPE time) per key frame.

        source index = stream frame index for window/current frames, slot index
        for memory slots (slot k covers stream frames [5k, 5k+5)).
        """
        return np.array([(p, f.index, t) for p, f, t in self.key_frames()], dtype=np.int64).reshape(-1, 3)

    @property
    def m(self) -> int:
        return len(self.memory)

    @property
    def w_frames(self) -> int:
        return len(self.window)

    # -- attend ------------------------------------------------------------
    def attend(self, q: np.ndarray, rows: Optional[Sequence[int]] = None, heads: Optional[Sequence[int]] = None,
               t_offset: int = 0) -> Tuple[np.ndarray, np.ndarray]:
        """Attention of the current block's queries over [memory | window | current].

        q: [b, T, H, D] exact query values (the block's own queries).
        rows: query rows r in [0, b*T) to evaluate (all if None); row r is
        token r % T of current frame r // T.
        t_offset: added to every time index (both queries and keys); the output
        must not depend on it (RoPE is relative).
        Returns (o[n, H', D], weight sums[n, H']) in float64.
        """
        cfg = self.cfg
        T, D = cfg.T, cfg.D
        b = q.shape[0]
        assert b == len(self.current), "attend() must follow the append of the same block"
        rows = np.arange(b * T) if rows is None else np.asarray(rows, dtype=np.int64)
        heads = list(range(cfg.H)) if heads is None else list(heads)
        kf = self.key_frames()
        tok = np.arange(T)
        ky, kx = tok // cfg.grid_w, tok % cfg.grid_w
        k_t = np.concatenate([np.full(T, t) for _, _, t in kf]) + t_offset
        k_y = np.tile(ky, len(kf))
        k_x = np.tile(kx, len(kf))
        qf, qs = rows // T, rows % T
        q_t = (len(self.sink) + self.m + self.w_frames + qf) + t_offset
        q_y, q_x = qs // cfg.grid_w, qs % cfg.grid_w
        split = cfg.rope()
        o = np.zeros((len(rows), len(heads), D))
        psum = np.zeros((len(rows), len(heads)))
        k_ang = rope_angles(k_t, k_y, k_x, split, cfg.theta)             # [Nk, D/2], shared by all heads
        q_ang = rope_angles(q_t, q_y, q_x, split, cfg.theta)             # [n, D/2]
        kc, ks, qc, qs_ = np.cos(k_ang), np.sin(k_ang), np.cos(q_ang), np.sin(q_ang)
        for hi, h in enumerate(heads):
            kh = np.concatenate([f.k[:, h, :] for _, f, _ in kf])
            vh = np.concatenate([f.v[:, h, :] for _, f, _ in kf])
            k_rot = rope_apply(kh, kc, ks)
            q_rot = rope_apply(np.asarray(q[qf, qs, h, :], dtype=np.float64), qc, qs_)
            o[:, hi, :], psum[:, hi] = attend_rows(q_rot, k_rot, vh)
        return o, psum

    def memory_slot(self, age: int) -> Tuple[np.ndarray, np.ndarray]:
        """Stored (K, V) of the memory slot `age` positions after the oldest."""
        f = self.memory[age]
        return f.k, f.v

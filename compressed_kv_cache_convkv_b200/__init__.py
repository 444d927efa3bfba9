"""ConvKV Memory attention step on NVIDIA B200 (sm_100a).

Thin ctypes binding over the C ABI in ``include/convkv.h`` (library
``lib/libconvkv.so``).  It only marshals arguments: every step of the path
(append, conv compression, reset-RoPE attention) runs in the library's CUDA
kernels.  PyTorch provides device memory and the stream.  There is no CPU
fallback: if the library is missing, every entry point raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field, replace
from typing import Optional, Tuple

from .configs import PRESETS, Workload  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
# the in-tree build; CONVKV_LIB names another build of the same sources (a variant
# compiled with other -D options), loaded in its place
LIB_PATH = os.environ.get("CONVKV_LIB") or os.path.join(_HERE, "lib", "libconvkv.so")

OK = 0
ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_BAD_ORDER, ERR_OOM, ERR_CUDA, ERR_DEVICE_TIMEOUT = -1, -2, -3, -4, -5, -6
ERR_SCRATCH_LIMIT = -7
NOALLOC_MAX_FRAME_HEADS = 4096
KV_BF16, KV_FP8_E4M3, KV_NVFP4 = 0, 1, 2
COMPRESS_CONV, COMPRESS_MEAN = 0, 1
FLAG_DRY_RUN, FLAG_HOST_IO = 1, 2
PART_MEMORY, PART_WINDOW, PART_CURRENT = 0, 1, 2

# every exported function of include/convkv.h: name -> (restype, argtypes)
_P = ctypes.c_void_p
_SIGNATURES = {
    "convkv_create": (ctypes.c_int, [_P, ctypes.POINTER(_P)]),
    "convkv_append_block": (ctypes.c_int, [_P, _P, _P, ctypes.c_int]),
    "convkv_attend": (ctypes.c_int, [_P, _P, _P]),
    "convkv_set_sink": (ctypes.c_int, [_P, _P, _P]),
    "convkv_append_block_sp": (ctypes.c_int, [_P, _P, _P, ctypes.c_int]),
    "convkv_attend_sp": (ctypes.c_int, [_P, _P, _P]),
    "convkv_ipc_export": (ctypes.c_int, [_P, _P, _P]),
    "convkv_ipc_open": (ctypes.c_int, [_P, _P]),
    "convkv_ipc_close": (ctypes.c_int, [_P]),
    "convkv_append_block_host": (ctypes.c_int, [_P, _P, _P, ctypes.c_int]),
    "convkv_attend_host": (ctypes.c_int, [_P, _P, _P]),
    "convkv_step_host": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int]),
    "convkv_step_host_async": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int]),
    "convkv_sync": (ctypes.c_int, [_P]),
    "convkv_state_bytes": (ctypes.c_size_t, [_P]),
    "convkv_destroy": (None, [_P]),
    "convkv_layout": (ctypes.c_int, [_P, _P, ctypes.c_int]),
    "convkv_host_chunks": (ctypes.c_int, [_P, ctypes.c_int, _P, ctypes.c_int]),
    "convkv_counters": (ctypes.c_int, [_P, _P]),
    "convkv_read_slot": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P]),
    "convkv_read_ring": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P]),
    "convkv_status": (ctypes.c_int, [_P]),
    "convkv_launch_count": (ctypes.c_int64, [_P]),
    "convkv_last_cuda_error": (ctypes.c_int, [_P]),
    "convkv_debug_fail_step": (ctypes.c_int, [_P, ctypes.c_int]),
    "convkv_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "convkv_quantize_e4m3_noalloc": (ctypes.c_int, [_P, _P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                    ctypes.c_int, _P]),
    "convkv_selftest_wait_timeout": (ctypes.c_int, [_P, ctypes.c_longlong, _P]),
    "convkv_selftest_div_rn": (ctypes.c_int, [_P, _P, ctypes.c_int64, _P, _P]),
}


class ConvKVError(RuntimeError):
    def __init__(self, code: int, what: str, cuda: int = 0):
        msg = f"{what}: {_lib().convkv_strerror(code).decode()} ({code})"
        if cuda:
            msg += f", cudaError {cuda}"
        super().__init__(msg)
        self.code = code


class _CCfg(ctypes.Structure):
    _fields_ = [
        ("heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
        ("first_block_frames", ctypes.c_int), ("block_frames", ctypes.c_int), ("window_frames", ctypes.c_int),
        ("evict_frames", ctypes.c_int), ("mem_slots", ctypes.c_int), ("rope_t", ctypes.c_int),
        ("rope_h", ctypes.c_int), ("rope_w", ctypes.c_int), ("rope_theta", ctypes.c_double),
        ("kv_format", ctypes.c_int), ("compress_mode", ctypes.c_int), ("num_states", ctypes.c_int),
        ("flags", ctypes.c_int), ("t_offset", ctypes.c_int), ("conv_weight", ctypes.c_void_p),
        ("stream", ctypes.c_void_p), ("sink_frames", ctypes.c_int), ("sp_ranks", ctypes.c_int),
        ("sp_rank", ctypes.c_int),
    ]


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} (run compressed_kv_cache_convkv_b200.build.build())")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def library():
    """The loaded ctypes library (raises if it is not built)."""
    return _lib()


def quantize_e4m3_noalloc(x, codes, scales, stream=None) -> None:
    """e4m3 codes and per-(frame, head) scales of bf16 frames x[frames, tokens, heads, head_dim],
    written into the caller's `codes` (uint8, same shape) and `scales` (float32 [frames, heads]),
    without any device allocation (for callers that cannot allocate while they run).  Calls that
    overlap on the GPU share one fixed scratch array and race."""
    import torch
    f, t, h, d = x.shape
    if x.dtype != torch.bfloat16 or codes.dtype != torch.uint8 or scales.dtype != torch.float32 or \
            tuple(codes.shape) != (f, t, h, d) or tuple(scales.shape) != (f, h) or \
            not (x.is_contiguous() and codes.is_contiguous() and scales.is_contiguous()):
        raise ValueError("x bf16 [F,T,H,D], codes uint8 [F,T,H,D], scales float32 [F,H], all contiguous")
    s = (stream or torch.cuda.current_stream()).cuda_stream
    rc = _lib().convkv_quantize_e4m3_noalloc(x.data_ptr(), codes.data_ptr(), scales.data_ptr(), f, t, h, d, s)
    if rc != OK:
        raise ConvKVError(rc, "convkv_quantize_e4m3_noalloc")


@dataclass
class Config:
    heads: int
    head_dim: int
    grid_h: int
    grid_w: int
    first_block_frames: int
    block_frames: int
    window_frames: int
    mem_slots: int
    evict_frames: int = 5
    rope: Tuple[int, int, int] = (0, 0, 0)
    rope_theta: float = 1e4
    kv_format: int = KV_BF16
    compress_mode: int = COMPRESS_CONV
    num_states: int = 1
    dry_run: bool = False
    host_io: bool = False
    t_offset: int = 0
    sink_frames: int = 0
    sp_ranks: int = 1       # sequence-parallel group size; `heads` is then this rank's share
    sp_rank: int = 0

    @property
    def T(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def max_block(self) -> int:
        return max(self.first_block_frames, self.block_frames)

    @property
    def ring_frames(self) -> int:
        return self.window_frames + self.max_block

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)

    def _c(self, conv_weight_ptr: int, stream_ptr: int) -> _CCfg:
        c = _CCfg()
        for name in ("heads", "head_dim", "grid_h", "grid_w", "first_block_frames", "block_frames",
                     "window_frames", "evict_frames", "mem_slots", "rope_theta", "kv_format", "compress_mode",
                     "num_states", "t_offset", "sink_frames", "sp_ranks", "sp_rank"):
            setattr(c, name, getattr(self, name))
        c.rope_t, c.rope_h, c.rope_w = self.rope
        c.flags = (FLAG_DRY_RUN if self.dry_run else 0) | (FLAG_HOST_IO if self.host_io else 0)
        c.conv_weight = conv_weight_ptr or None
        c.stream = stream_ptr or None
        return c


class ConvKV:
    """One ConvKV cache (``num_states`` independent states advanced together).

    Per block: ``append(k, v)`` then ``attend(q)``.  Tensors are bf16 CUDA
    tensors of shape [num_states, frames*T, H, D] (or [frames*T, H, D] when
    num_states == 1), contiguous.  All work runs on the stream that was
    current when the cache was created.
    """

    def __init__(self, cfg: Config, conv_weight=None, stream=None):
        import torch
        self.cfg = cfg
        self._h = ctypes.c_void_p()
        wptr = 0
        if conv_weight is not None:
            S, H, D = cfg.num_states, cfg.heads, cfg.head_dim
            want = (S, 2, H, D, D, 5)
            w = conv_weight.reshape(want) if conv_weight.numel() == S * 2 * H * D * D * 5 else None
            if w is None or conv_weight.dtype != torch.bfloat16 or not conv_weight.is_cuda or \
                    not conv_weight.is_contiguous():
                raise ValueError(f"conv_weight must be a contiguous bf16 CUDA tensor with shape {want}")
            wptr = conv_weight.data_ptr()
        if stream is None and not cfg.dry_run:
            stream = torch.cuda.current_stream()
        self._stream = stream
        sptr = stream.cuda_stream if stream is not None else 0
        c = cfg._c(wptr, sptr)
        rc = _lib().convkv_create(ctypes.byref(c), ctypes.byref(self._h))
        if rc != OK:
            self._h = ctypes.c_void_p()
            raise ConvKVError(rc, "convkv_create")

    # -- lifecycle ----------------------------------------------------------
    def close(self) -> None:
        if self._h:
            _lib().convkv_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, rc: int, what: str) -> None:
        if rc != OK:
            raise ConvKVError(rc, what, _lib().convkv_last_cuda_error(self._h))

    def _frames_of(self, x, name: str) -> int:
        import torch
        cfg = self.cfg
        if x.dtype != torch.bfloat16 or not x.is_contiguous():
            raise ValueError(f"{name} must be contiguous bf16")
        shape = tuple(x.shape)
        if cfg.num_states == 1 and len(shape) == 3:
            shape = (1,) + shape
        if len(shape) != 4 or shape[0] != cfg.num_states or shape[2] != cfg.heads or shape[3] != cfg.head_dim \
                or shape[1] % cfg.T:
            raise ValueError(f"{name} has shape {tuple(x.shape)}; want [{cfg.num_states}, frames*{cfg.T}, "
                             f"{cfg.heads}, {cfg.head_dim}]")
        return shape[1] // cfg.T

    # -- the step -----------------------------------------------------------
    def append(self, k, v) -> None:
        fk, fv = self._frames_of(k, "k"), self._frames_of(v, "v")
        if fk != fv:
            raise ValueError("k and v must carry the same number of frames")
        if not (k.is_cuda and v.is_cuda):
            raise ValueError("k, v must be CUDA tensors (use append_host for host buffers)")
        self._check(_lib().convkv_append_block(self._h, k.data_ptr(), v.data_ptr(), fk), "convkv_append_block")

    def attend(self, q, out=None):
        import torch
        self._frames_of(q, "q")
        if out is None:
            out = torch.empty_like(q)
        self._check(_lib().convkv_attend(self._h, q.data_ptr(), out.data_ptr()), "convkv_attend")
        return out

    def set_sink(self, k, v) -> None:
        """K/V of the ``sink_frames`` reference frames, attended first by every block and
        never evicted; bf16 CUDA tensors [num_states, sink_frames*T, H, D]."""
        if self.cfg.dry_run:
            self._check(_lib().convkv_set_sink(self._h, None, None), "convkv_set_sink")
            return
        fk, fv = self._frames_of(k, "k"), self._frames_of(v, "v")
        if fk != self.cfg.sink_frames or fv != fk or not (k.is_cuda and v.is_cuda):
            raise ValueError(f"k, v must be CUDA tensors of {self.cfg.sink_frames} reference frames")
        self._check(_lib().convkv_set_sink(self._h, k.data_ptr(), v.data_ptr()), "convkv_set_sink")

    # -- sequence-parallel forms: the all-to-all is fused into the kernels ----
    def _ptrs(self, shards, name):
        if len(shards) != self.cfg.sp_ranks:
            raise ValueError(f"{name}: want {self.cfg.sp_ranks} shards, got {len(shards)}")
        return (ctypes.c_void_p * len(shards))(*[t.data_ptr() for t in shards])

    def append_sp(self, k_shards, v_shards, frames: int) -> None:
        """k_shards[r], v_shards[r]: rank r's rows of the block (every head), bf16 CUDA
        tensors [num_states, rows_r, sp_ranks*heads, D] with rows_r from shard_rows()."""
        self._check(_lib().convkv_append_block_sp(self._h, self._ptrs(k_shards, "k"), self._ptrs(v_shards, "v"),
                                                  frames), "convkv_append_block_sp")

    def attend_sp(self, q_shards, out_shards) -> None:
        """Queries from, and outputs into, the ranks' sequence shards (same layout as append_sp)."""
        self._check(_lib().convkv_attend_sp(self._h, self._ptrs(q_shards, "q"), self._ptrs(out_shards, "out")),
                    "convkv_attend_sp")

    def append_host(self, k, v) -> None:
        fk = self._frames_of(k, "k")
        self._check(_lib().convkv_append_block_host(self._h, k.data_ptr(), v.data_ptr(), fk),
                    "convkv_append_block_host")

    def attend_host(self, q, out) -> None:
        self._frames_of(q, "q")
        self._check(_lib().convkv_attend_host(self._h, q.data_ptr(), out.data_ptr()), "convkv_attend_host")

    def _step_frames(self, k, v, q) -> int:
        fk, fq = self._frames_of(k, "k"), self._frames_of(q, "q")
        if fk != self._frames_of(v, "v") or fk != fq:
            raise ValueError("k, v and q must carry the same number of frames")
        return fk

    def step_host(self, k, v, q, out) -> None:
        """append_host(k, v) then attend_host(q, out) as one pipelined call (host buffers,
        pinned for overlap): per chunk, copies in, ring append, attention and the copy
        back overlap the other chunks'."""
        fk = self._step_frames(k, v, q)
        self._check(_lib().convkv_step_host(self._h, k.data_ptr(), v.data_ptr(), q.data_ptr(), out.data_ptr(), fk),
                    "convkv_step_host")

    def step_host_async(self, k, v, q, out) -> None:
        """step_host, returned once queued: the next step's copies overlap this step's
        kernels.  Keep the buffers alive and unchanged (out unread) until sync()."""
        fk = self._step_frames(k, v, q)
        self._check(_lib().convkv_step_host_async(self._h, k.data_ptr(), v.data_ptr(), q.data_ptr(),
                                                  out.data_ptr(), fk), "convkv_step_host_async")

    def sync(self) -> None:
        """Wait for every queued call of the handle (kernels and host copies)."""
        self._check(_lib().convkv_sync(self._h), "convkv_sync")

    def dry_append(self, frames: int) -> None:
        """Advance the bookkeeping only (dry-run handles)."""
        self._check(_lib().convkv_append_block(self._h, None, None, frames), "convkv_append_block")

    # -- introspection ------------------------------------------------------
    def state_bytes(self) -> int:
        return int(_lib().convkv_state_bytes(self._h))

    def launch_count(self) -> int:
        return int(_lib().convkv_launch_count(self._h))

    def counters(self) -> dict:
        buf = (ctypes.c_int64 * 8)()
        self._check(_lib().convkv_counters(self._h, buf), "convkv_counters")
        keys = ("P", "E", "S", "m", "w", "b", "blocks", "groups")
        return dict(zip(keys, (int(x) for x in buf)))

    def layout(self):
        import numpy as np
        n = _lib().convkv_layout(self._h, None, 0)
        if n < 0:
            raise ConvKVError(n, "convkv_layout")
        rec = np.zeros((max(n, 1), 4), dtype=np.int32)
        _lib().convkv_layout(self._h, rec.ctypes.data, n)
        return rec[:n]

    def host_chunks(self, queued: bool = False):
        """The host-buffer chunk plan: rows of (first state, states, first head, heads);
        queued: the plan of a queued step that follows a queued step."""
        import numpy as np
        n = _lib().convkv_host_chunks(self._h, int(queued), None, 0)
        if n < 0:
            raise ConvKVError(n, "convkv_host_chunks")
        rec = np.zeros((max(n, 1), 4), dtype=np.int32)
        _lib().convkv_host_chunks(self._h, int(queued), rec.ctypes.data, n)
        return rec[:n]

    def _read(self, fn, name: str, state: int, kv: int, idx: int):
        import numpy as np
        cfg = self.cfg
        T, H, D = cfg.T, cfg.heads, cfg.head_dim
        sc = np.zeros(H, dtype=np.float32)
        if cfg.kv_format == KV_NVFP4:
            raw = np.zeros(T * H * D // 2 + T * H * D // 16, dtype=np.uint8)
            self._check(fn(self._h, state, kv, idx, raw.ctypes.data, sc.ctypes.data), name)
            n = T * H * D // 2
            return raw[:n].reshape(T, H, D // 2), (raw[n:].reshape(T, H, D // 16), sc)
        dt = np.uint8 if cfg.kv_format == KV_FP8_E4M3 else np.uint16
        dst = np.zeros((T, H, D), dtype=dt)
        self._check(fn(self._h, state, kv, idx, dst.ctypes.data, sc.ctypes.data), name)
        return dst, (sc if cfg.kv_format == KV_FP8_E4M3 else None)

    def read_slot(self, state: int, kv: int, pos: int):
        """Memory position `pos`: (bf16 bits [T, H, D] as uint16, None); in the fp8 format
        (e4m3 codes uint8 [T, H, D], scales[H]); in the NVFP4 format (e2m1 pairs uint8
        [T, H, D/2], (e4m3 block scales uint8 [T, H, D/16], scales[H]))."""
        return self._read(_lib().convkv_read_slot, "convkv_read_slot", state, kv, pos)

    def read_ring(self, state: int, kv: int, slot: int):
        """Same as read_slot for ring slot `slot`."""
        return self._read(_lib().convkv_read_ring, "convkv_read_ring", state, kv, slot)

    def status(self) -> int:
        return int(_lib().convkv_status(self._h))

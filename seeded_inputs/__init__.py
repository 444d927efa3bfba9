"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module holds none of the ConvKV method's arithmetic.  It maps
(seed, tensor, state, frame, element) to one bf16 value with a counter-based
generator (Philox4x32-10) and an integer-exact Irwin-Hall(12) transform, so
that the same value can be produced on the host (for the oracle) and on the
device (for long streams that never leave HBM) bit for bit.

Tensor ids and element order:
  Q, K, V  : frame = stream latent-frame index, element = (s*H + h)*D + d
             for token s of the frame, head h, channel d  ([T][H][D] per frame)
  WK, WV   : frame = 0, element = ((h*D + o)*D + i)*5 + j
             ([H][D_out][D_in][5] conv weights, scaled by 1/sqrt(5*D))
  RK, RV   : frame = reference-image frame index, element as for K and V
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

Q, K, V, WK, WV, RK, RV = 0, 1, 2, 3, 4, 5, 6

_HERE = os.path.dirname(os.path.abspath(__file__))
_HOST_SO = os.path.join(_HERE, "libseeded_inputs_host.so")
_DEV_SO = os.path.join(_HERE, "libseeded_inputs_cuda.so")
_host = None
_dev = None


def build(device: bool = True) -> None:
    """Compile the host generator (gcc) and, if asked, the device one (nvcc, sm_100a)."""
    src = os.path.join(_HERE, "gen_host.c")
    if _stale(_HOST_SO, src):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-o", _HOST_SO, src])
    if device:
        dsrc = os.path.join(_HERE, "gen_device.cu")
        if _stale(_DEV_SO, dsrc):
            subprocess.check_call(["nvcc", "-O3", "-shared", "-Xcompiler", "-fPIC",
                                   "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                                   "-fmad=false", "-o", _DEV_SO, dsrc])


def _stale(out: str, src: str) -> bool:
    return (not os.path.exists(out)) or os.path.getmtime(out) < os.path.getmtime(src)


def _host_lib():
    global _host
    if _host is None:
        build(device=False)
        lib = ctypes.CDLL(_HOST_SO)
        lib.si_fill_bf16.argtypes = [ctypes.c_void_p, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32,
                                     ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_float]
        lib.si_fill_bf16.restype = None
        lib.si_fill_bf16_indexed.argtypes = [ctypes.c_void_p, ctypes.c_uint32, ctypes.c_uint32,
                                             ctypes.c_uint32, ctypes.c_uint32, ctypes.c_void_p,
                                             ctypes.c_int64, ctypes.c_float]
        lib.si_fill_bf16_indexed.restype = None
        lib.si_philox4x32_10.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.si_philox4x32_10.restype = None
        _host = lib
    return _host


def _dev_lib():
    global _dev
    if _dev is None:
        if not os.path.exists(_DEV_SO):
            raise RuntimeError(f"device input generator not built: {_DEV_SO} (run seeded_inputs.build())")
        lib = ctypes.CDLL(_DEV_SO)
        lib.si_fill_bf16_device.argtypes = [ctypes.c_void_p, ctypes.c_uint32, ctypes.c_uint32,
                                            ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32,
                                            ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p]
        lib.si_fill_bf16_device.restype = ctypes.c_int
        _dev = lib
    return _dev


def philox4x32_10(ctr, key) -> tuple:
    """Raw generator output for one counter/key (used by known-answer tests)."""
    c = (ctypes.c_uint32 * 4)(*ctr)
    k = (ctypes.c_uint32 * 2)(*key)
    o = (ctypes.c_uint32 * 4)()
    _host_lib().si_philox4x32_10(c, k, o)
    return tuple(int(x) for x in o)


def weight_scale(D: int) -> float:
    """fp32 scale that turns the unit-variance values into N(0, 1/(5*D)) conv weights."""
    return float(np.float32(1.0 / math.sqrt(5.0 * D)))


def frames(seed: int, tensor: int, state: int, frame0: int, nframes: int, frame_elems: int,
           scale: float = 1.0) -> np.ndarray:
    """bf16 bit patterns (uint16) of shape [nframes, frame_elems]."""
    out = np.empty((nframes, frame_elems), dtype=np.uint16)
    if out.size:
        _host_lib().si_fill_bf16(out.ctypes.data, seed, tensor, state, frame0, nframes, frame_elems, scale)
    return out


def frame_elements(seed: int, tensor: int, state: int, frame: int, elems: np.ndarray,
                   scale: float = 1.0) -> np.ndarray:
    """bf16 bit patterns at the given element indices of one frame."""
    idx = np.ascontiguousarray(elems, dtype=np.uint32)
    out = np.empty(idx.shape, dtype=np.uint16)
    if idx.size:
        _host_lib().si_fill_bf16_indexed(out.ctypes.data, seed, tensor, state, frame,
                                          idx.ctypes.data, idx.size, scale)
    return out


def conv_weights(seed: int, state: int, H: int, D: int) -> np.ndarray:
    """bf16 bits [2(K,V), H, D_out, D_in, 5]."""
    n = H * D * D * 5
    wk = frames(seed, WK, state, 0, 1, n, weight_scale(D))
    wv = frames(seed, WV, state, 0, 1, n, weight_scale(D))
    return np.stack([wk.reshape(H, D, D, 5), wv.reshape(H, D, D, 5)])


def frames_device(ptr: int, seed: int, tensor: int, state: int, frame0: int, nframes: int,
                  frame_elems: int, scale: float = 1.0, stream: int = 0) -> None:
    """Same values as frames(), written to device memory at ptr on `stream`."""
    rc = _dev_lib().si_fill_bf16_device(ptr, seed, tensor, state, frame0, nframes, frame_elems,
                                        scale, stream)
    if rc != 0:
        raise RuntimeError(f"si_fill_bf16_device failed: cudaError {rc}")


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)

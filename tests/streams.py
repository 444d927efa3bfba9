"""Drive one workload through the CUDA path and the oracle on the same seeded inputs.

Inputs for block n are frames [F_n, F_n + b_n) of the seeded Q, K, V tensors
(SoulX-style streams: stream frame index = latent frame index), generated on
the device for the CUDA path and on the host for the oracle, bit-identical.
"""
from __future__ import annotations

import math
from typing import Iterator, Optional, Sequence

import numpy as np

import seeded_inputs as si
from oracle import convkv_oracle as O

# tolerances (the target bounds; relative form for compressed K/V of magnitude > 1,
# plus a relative-L2 gate on attention outputs whose magnitude is ~1e-2)
ATT_MAX, ATT_MEAN, ATT_REL_L2 = 1e-2, 1e-3, 1e-2
SLOT_MAX_REL, SLOT_MEAN = 1e-2, 1e-3
FP8_MAX = 5e-2


def oracle_for(w, state: int = 0, conv_w: Optional[np.ndarray] = None, mean: bool = False,
               heads: Optional[Sequence[int]] = None) -> O.OracleStream:
    """Oracle state of workload w, for every head or only `heads` (heads are independent
    through the whole step: conv weights, quantisation scales and attention are per head,
    so a head subset gives exactly the values of those heads)."""
    H = w.heads if heads is None else len(heads)
    cfg = O.OracleConfig(H=H, D=w.head_dim, grid_h=w.grid_h, grid_w=w.grid_w, window=w.window_frames,
                         mem_slots=w.mem_slots, fp8=w.fp8, fp4=getattr(w, "fp4", False))
    if mean:
        wts = np.zeros((2, H, w.head_dim, w.head_dim, 5))
        for o in range(w.head_dim):
            wts[:, :, o, o, :] = 0.2
    else:
        wts = si.bf16_bits_to_f64(conv_w if conv_w is not None else si.conv_weights(w.seed, state, w.heads, w.head_dim))
        if heads is not None:
            wts = wts[:, list(heads)]
    return O.OracleStream(cfg, wts)


def host_frames(w, tensor: int, state: int, frame0: int, nframes: int,
                heads: Optional[Sequence[int]] = None) -> np.ndarray:
    """bf16 bits [nframes, T, H', D] of the seeded frames, every head or only `heads`."""
    fe = w.T * w.heads * w.head_dim
    if heads is None:
        return si.frames(w.seed, tensor, state, frame0, nframes, fe).reshape(nframes, w.T, w.heads, w.head_dim)
    hs = np.asarray(list(heads), dtype=np.int64)
    idx = ((np.arange(w.T)[:, None, None] * w.heads + hs[None, :, None]) * w.head_dim
           + np.arange(w.head_dim)[None, None, :]).reshape(-1)
    out = np.stack([si.frame_elements(w.seed, tensor, state, frame0 + f, idx) for f in range(nframes)])
    return out.reshape(nframes, w.T, len(hs), w.head_dim)


def select_heads(x, heads: Optional[Sequence[int]], axis: int = 1):
    """x restricted to `heads` along `axis` (x itself when heads is None)."""
    if heads is None:
        return x
    return np.take(x, list(heads), axis=axis)


def device_frames(w, tensor: int, frame0: int, nframes: int, torch_mod, out=None):
    """[S, nframes*T, H, D] bf16 CUDA tensor of the seeded values (all states)."""
    torch = torch_mod
    S = w.num_states
    fe = w.T * w.heads * w.head_dim
    if out is None:
        out = torch.empty((S, nframes * w.T, w.heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for s in range(S):
        si.frames_device(out[s].data_ptr(), w.seed, tensor, s, frame0, nframes, fe, 1.0, stream)
    return out


def device_weights(w, torch_mod, states: Optional[Sequence[int]] = None):
    torch = torch_mod
    S = w.num_states
    n = w.heads * w.head_dim * w.head_dim * 5
    out = torch.empty((S, 2, w.heads, w.head_dim, w.head_dim, 5), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for s in range(S):
        for kv, tid in ((0, si.WK), (1, si.WV)):
            si.frames_device(out[s, kv].data_ptr(), w.seed, tid, s, 0, 1, n, si.weight_scale(w.head_dim), stream)
    return out


def bf16_tensor_to_f64(t) -> np.ndarray:
    import torch
    return si.bf16_bits_to_f64(t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def sample_rows(w, b: int, n: int, rng: np.random.Generator) -> np.ndarray:
    """Query rows to check: first/last rows, the ragged tail of the last 128-row tile, random rest."""
    Nq = b * w.T
    if n >= Nq:
        return np.arange(Nq)
    fixed = {0, 1, Nq - 1, Nq - 2, w.T - 1, w.T}
    tail0 = (Nq // 128) * 128
    fixed |= set(range(tail0, min(Nq, tail0 + 4)))
    fixed |= {r for r in range(127, Nq, 128)}
    fixed = sorted(x for x in fixed if 0 <= x < Nq)[: n // 2]
    rest = rng.choice(Nq, size=n - len(fixed), replace=False)
    return np.unique(np.concatenate([np.array(fixed, dtype=np.int64), rest]))


def attention_errors(gpu: np.ndarray, ref: np.ndarray) -> dict:
    d = np.abs(gpu - ref)
    return {"max": float(d.max()), "mean": float(d.mean()),
            "rel_l2": float(np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300))}


# Sharp-softmax variant (queries x8, outputs of order 1): the bf16 rounding of the
# rotated operands (relative 2^-9 each) moves a logit of size ~8 by ~0.03, i.e. a few
# percent on the weights of competing keys, so the absolute bound scales with it.
SHARP_MAX, SHARP_MEAN = 6e-2, 5e-3


def check_attention(gpu: np.ndarray, ref: np.ndarray, fp8: bool = False, what: str = "", sharp: bool = False) -> dict:
    e = attention_errors(gpu, ref)
    if sharp:
        assert e["max"] <= SHARP_MAX and e["mean"] <= SHARP_MEAN and e["rel_l2"] <= ATT_REL_L2, (what, e)
    elif fp8:
        assert e["max"] <= FP8_MAX and e["rel_l2"] <= 5 * ATT_REL_L2, (what, e)
    else:
        assert e["max"] <= ATT_MAX and e["mean"] <= ATT_MEAN and e["rel_l2"] <= ATT_REL_L2, (what, e)
    return e


# Heavy-tailed inputs (a few x16 values per frame and head in K and V): logits are no
# longer unit-variance and a row can be dominated by one key, whose value may itself be
# an outlier.  The bf16 rounding of the rotated operands moves a logit by ~2^-8 of the
# sum of |q_d k_d| / sqrt(D), and the output by that much of the spread of V across the
# dominant keys, so the sharp-softmax bound applies, scaled by the size of the output.
OUTLIER_MAX_REL, OUTLIER_REL_L2 = 6e-2, 5e-2


def check_attention_scaled(gpu: np.ndarray, ref: np.ndarray, what: str = "") -> dict:
    d = np.abs(gpu - ref)
    e = {"max_rel": float((d / np.maximum(1.0, np.abs(ref))).max()),
         "rel_l2": float(np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300))}
    assert e["max_rel"] <= OUTLIER_MAX_REL and e["rel_l2"] <= OUTLIER_REL_L2, (what, e)
    return e


def check_slot(gpu: np.ndarray, ref: np.ndarray, what: str = "") -> dict:
    d = np.abs(gpu - ref)
    rel = d / np.maximum(1.0, np.abs(ref))
    e = {"max_rel": float(rel.max()), "mean": float(d.mean())}
    assert e["max_rel"] <= SLOT_MAX_REL and e["mean"] <= SLOT_MEAN, (what, e)
    return e


def e4m3_bytes_to_f64(b: np.ndarray) -> np.ndarray:
    """Values of e4m3 codes (uint8 bit patterns)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(b, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


E4M3_CODE_MISMATCH = 1e-3   # fraction of conv-output codes allowed to sit one step apart


def check_codes(gpu_bytes: np.ndarray, gpu_scales: np.ndarray, ref_codes: np.ndarray, ref_scales: np.ndarray,
                exact: bool, what: str = "") -> dict:
    """e4m3 codes and per-head scales against the oracle's.

    exact: bit-exact (quantised from identical bf16 inputs with the same fp32
    arithmetic).  Otherwise (quantised conv outputs, fp32 accumulation on the GPU
    against fp64 in the oracle): scales within 1e-5 relative, codes equal except
    for a small fraction one quantisation step apart (values next to a rounding
    boundary)."""
    g = e4m3_bytes_to_f64(gpu_bytes)
    if exact:
        assert np.array_equal(gpu_scales, ref_scales.astype(np.float32)), (what, "scales")
        assert np.array_equal(g, ref_codes), (what, "codes", int(np.sum(g != ref_codes)))
        return {"mismatch": 0.0}
    rs = np.abs(gpu_scales.astype(np.float64) / ref_scales.astype(np.float64) - 1).max()
    assert rs <= 1e-5, (what, "scale", rs)
    diff = g != ref_codes
    frac = float(diff.mean())
    assert frac <= E4M3_CODE_MISMATCH, (what, "code mismatch fraction", frac)
    if diff.any():
        a = np.abs(ref_codes[diff])
        _, ex = np.frexp(np.where(a > 0, a, 1.0))
        step = np.exp2(np.maximum(ex - 1.0, -6.0) - 3.0)      # e4m3 quantum at the reference value
        assert np.all(np.abs(g[diff] - ref_codes[diff]) <= step * 2 + 1e-30), (what, "code step")
    return {"mismatch": frac}


# -- NVFP4 ------------------------------------------------------------------

E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_pairs_to_f64(pairs: np.ndarray) -> np.ndarray:
    """bytes [..., D/2] of e2m1 pairs (even channel in the low nibble) -> values [..., D]."""
    b = np.asarray(pairs, dtype=np.uint8)
    nib = np.stack([b & 0xF, b >> 4], axis=-1).reshape(*b.shape[:-1], b.shape[-1] * 2)
    val = E2M1_VALUES[nib & 7]
    return np.where(nib & 8, -val, val)


def fp4_values(codes: np.ndarray, bs: np.ndarray, g: np.ndarray) -> np.ndarray:
    """code * fp32(s_b * g) in fp32, for values [T, H, D], block scales [T, H, D/16], g[H]."""
    T, H, D = codes.shape
    eb = (np.asarray(bs, np.float32) * np.asarray(g, np.float32)[None, :, None]).astype(np.float32)
    return (codes.astype(np.float32).reshape(T, H, D // 16, 16) * eb[..., None]).astype(np.float32).reshape(T, H, D)


def check_codes_fp4(gpu, ref, exact: bool, what: str = "", max_frac: float = 0.0) -> dict:
    """gpu = (e2m1 pair bytes [T, H, D/2], (e4m3 block scale bytes [T, H, D/16], g[H]));
    ref = (code values [T, H, D], (block scale values [T, H, D/16], g[H])) from the oracle.

    exact: every code, block scale and tensor scale equal.  Otherwise (quantised conv
    outputs: fp32 accumulation on the GPU against fp64 in the oracle) tensor scales
    within 1e-5 relative, and the fraction of channels whose dequantised value differs
    by more than that at most max_frac; such a value is within one e2m1 step at the
    larger of the two block scales (values next to a rounding boundary, of a code or
    of its block's scale)."""
    gc, (gb, gg) = gpu
    rc, (rb, rg) = ref
    gcv = e2m1_pairs_to_f64(gc)
    gbv = e4m3_bytes_to_f64(gb)
    if exact:
        assert np.array_equal(gg, np.asarray(rg, np.float32)), (what, "tensor scales")
        assert np.array_equal(gbv, rb), (what, "block scales", int(np.sum(gbv != rb)))
        assert np.array_equal(gcv, rc), (what, "codes", int(np.sum(gcv != rc)))
        return {"mismatch": 0.0}
    rs = np.abs(gg.astype(np.float64) / np.asarray(rg, np.float64) - 1).max()
    assert rs <= 1e-5, (what, "tensor scale", rs)
    gv, rv = fp4_values(gcv, gbv, gg), fp4_values(rc, rb, rg)
    # same code and block scale: the values differ only through g (<= 1e-5 relative)
    diff = np.abs(gv.astype(np.float64) - rv) > 2e-5 * np.abs(rv)
    frac = float(diff.mean())
    assert frac <= max_frac, (what, "value mismatch fraction", frac)
    if diff.any():
        T, H, D = rc.shape
        eg = (gbv.astype(np.float32) * gg[None, :, None]).repeat(16, axis=2)
        er = (rb.astype(np.float32) * np.asarray(rg, np.float32)[None, :, None]).repeat(16, axis=2)
        step = 2.0 * np.maximum(eg, er)                      # the largest e2m1 step is 2 (between 4 and 6)
        assert np.all(np.abs(gv - rv)[diff] <= step[diff] * 1.0001 + 1e-30), (what, "value step")
    return {"mismatch": frac, "block_scale_mismatch": float((gbv != rb).mean())}

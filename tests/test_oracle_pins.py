"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test checks one oracle function against a closed form, a library routine,
a hand-derived table or an invariant the mathematics fixes, chosen so that a
plausible mistake (dropped term, wrong sign, transposed operand, wrong index,
off-by-one in the eviction rule) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import convkv_oracle as O

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- rounding

def test_round_to_bf16_matches_torch_cast():
    # fp32 inputs: torch's fp32 -> bf16 cast is a single round-to-nearest-even
    # (its fp64 -> bf16 cast goes through fp32 and can round twice)
    x = (RNG.standard_normal(200000) * np.exp(RNG.uniform(-20, 20, 200000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_to_bf16(x.astype(np.float64)), ref)
    # a value just below a halfway point must not be rounded up (single rounding)
    y = float.fromhex("0x1.72ffffdb61393p+0")
    assert O.round_to_bf16(np.array([y]))[0] == 1.4453125


def test_round_to_bf16_ties_to_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties go to the even mantissa (1.0)
    assert O.round_to_bf16(np.array([1 + 2 ** -8]))[0] == 1.0
    assert O.round_to_bf16(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6


def test_e4m3_matches_torch_cast_in_range():
    x = (RNG.standard_normal(300000) * np.exp(RNG.uniform(-12, 6.0, 300000))).astype(np.float32)
    x = x[np.abs(x) < 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(O.e4m3_rne_satfinite(x), ref)


def test_e4m3_saturates_and_known_values():
    v = O.e4m3_rne_satfinite(np.array([448, 460, 464, 1e6, -1e6, 2 ** -9, 2 ** -10, 3 * 2 ** -10, 0.0],
                                      dtype=np.float32))
    # 464 is halfway between 448 and 480 (not finite): ties-to-even gives 448; beyond: saturate
    assert list(v[:5]) == [448, 448, 448, 448, -448]
    assert v[5] == 2 ** -9           # smallest subnormal
    assert v[6] == 0.0               # halfway between 0 and 2^-9 -> even (0)
    assert v[7] == 2 * 2 ** -9       # 1.5 quanta -> 2 (even)
    assert v[8] == 0.0


def test_e4m3_grid_round_trip():
    # every finite e4m3 value is a fixed point of the quantiser
    vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    vals = vals[np.isfinite(vals)]
    assert np.array_equal(O.e4m3_rne_satfinite(vals), vals.astype(np.float64))


def test_fp8_dequantise_is_bf16_of_fp32_product():
    # "dequantize to BF16 on use": the consumed value is bf16(fp32(code * scale)); checked
    # against torch's own e4m3 decode, fp32 multiply and single-rounding fp32 -> bf16 cast
    x = RNG.standard_normal((32, 2, 16)) * 3
    code, scale = O.fp8_encode(x)
    deq = O.fp8_dequantize(code, scale)
    t = torch.from_numpy(code.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float32)
    ref = (t * torch.from_numpy(scale)[None, :, None]).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(deq, ref)


def test_fp8_quantize_scale_rule():
    x = RNG.standard_normal((16, 3, 8))
    x[:, 2, :] = 0.0
    deq, scale = O.fp8_quantize(x)
    amax = np.abs(x.astype(np.float32)).max(axis=(0, 2))
    assert scale[0] == np.float32(amax[0] / np.float32(448.0))
    assert scale[2] == 1.0 and np.all(deq[:, 2, :] == 0)
    # the largest-magnitude element of each head maps to +-448 * scale (up to the fp32 divide)
    for h in range(2):
        i = np.unravel_index(np.argmax(np.abs(x[:, h, :])), x[:, h, :].shape)
        assert abs(abs(deq[i[0], h, i[1]]) / scale[h] - 448) <= 32
    # dequantised error: half an e4m3 quantum (relative 2^-4) plus the bf16 rounding (2^-8)
    rel = np.abs(deq[:, :2] - x[:, :2].astype(np.float32)) / np.maximum(np.abs(x[:, :2]), 2 ** -6 * scale[:2][None, :, None])
    assert rel.max() <= 2 ** -4 + 2 ** -8 + 1e-6


# ---------------------------------------------------------------- RoPE

def test_rope_split_values():
    assert O.rope_split(128) == (44, 42, 42)
    assert O.rope_split(64) == (24, 20, 20)


def test_rope_hand_values():
    # D=6 split (2,2,2): one pair per axis, frequency theta^0 = 1 -> angle = position
    x = np.array([1.0, 0.0, 0.0, 1.0, 1.0, 1.0])
    out = O.rope_rotate(x, np.pi / 2, np.pi, np.pi / 4, (2, 2, 2), 1e4)
    np.testing.assert_allclose(out, [0.0, 1.0, 0.0, -1.0, 0.0, math.sqrt(2)], atol=1e-15)


def test_rope_frequency_hand_values():
    # time axis width 44, pair 11: theta^(-22/44) = 1e4^-0.5 = 0.01 -> t=100 turns by 1 rad
    x = np.zeros(128); x[22] = 1.0
    out = O.rope_rotate(x, 100.0, 0.0, 0.0, (44, 42, 42), 1e4)
    assert abs(out[22] - math.cos(1.0)) < 1e-13 and abs(out[23] - math.sin(1.0)) < 1e-13
    # row axis (channels 44..85), pair 7: theta^(-14/42) with theta=1e6 -> 0.01
    x = np.zeros(128); x[44 + 14] = 1.0
    out = O.rope_rotate(x, 0.0, 100.0, 0.0, (44, 42, 42), 1e6)
    assert abs(out[58] - math.cos(1.0)) < 1e-13 and abs(out[59] - math.sin(1.0)) < 1e-13
    # column axis (channels 86..127), pair 0 turns by the column index itself
    x = np.zeros(128); x[86] = 1.0
    out = O.rope_rotate(x, 0.0, 0.0, 2.0, (44, 42, 42), 1e4)
    assert abs(out[86] - math.cos(2.0)) < 1e-14 and abs(out[87] - math.sin(2.0)) < 1e-14


def _rope_complex(x, t, y, xc, split, theta):
    """Independent statement of the rotation as complex multiplication."""
    out = np.empty_like(x)
    start = 0
    for width, pos in zip(split, (t, y, xc)):
        z = x[..., start:start + width:2] + 1j * x[..., start + 1:start + width:2]
        freq = np.array([theta ** (-2.0 * i / width) for i in range(width // 2)])
        z = z * np.exp(1j * np.asarray(pos, dtype=np.float64)[..., None] * freq)
        out[..., start:start + width:2] = z.real
        out[..., start + 1:start + width:2] = z.imag
        start += width
    return out


def test_rope_matches_complex_form():
    x = RNG.standard_normal((50, 128))
    t, y, xc = RNG.integers(0, 40, 50), RNG.integers(0, 45, 50), RNG.integers(0, 52, 50)
    np.testing.assert_allclose(O.rope_rotate(x, t, y, xc, (44, 42, 42), 1e4),
                               _rope_complex(x, t, y, xc, (44, 42, 42), 1e4), rtol=0, atol=1e-12)


def test_rope_group_identities():
    x = RNG.standard_normal((20, 64))
    sp = O.rope_split(64)
    z = np.zeros(20)
    np.testing.assert_array_equal(O.rope_rotate(x, z, z, z, sp, 1e4), x)          # R(0) = I
    a = RNG.integers(0, 30, (3, 20)); b = RNG.integers(0, 30, (3, 20))
    ra = O.rope_rotate(x, *a, sp, 1e4)
    np.testing.assert_allclose(np.linalg.norm(ra, axis=1), np.linalg.norm(x, axis=1), rtol=1e-14)
    rab = O.rope_rotate(ra, *b, sp, 1e4)
    np.testing.assert_allclose(rab, O.rope_rotate(x, *(a + b), sp, 1e4), atol=1e-12)  # R(a)R(b)=R(a+b)


def test_rope_relative_scores():
    # <R(p)q, R(p')k> depends only on p - p' (the property RoPE Reset relies on)
    q, k = RNG.standard_normal(128), RNG.standard_normal(128)
    sp = (44, 42, 42)
    s1 = O.rope_rotate(q, 9, 3, 5, sp, 1e4) @ O.rope_rotate(k, 4, 1, 7, sp, 1e4)
    s2 = O.rope_rotate(q, 1009, 13, 25, sp, 1e4) @ O.rope_rotate(k, 1004, 11, 27, sp, 1e4)
    assert abs(s1 - s2) < 1e-10


# ---------------------------------------------------------------- conv

def test_conv_matches_torch_conv1d():
    T, H, D = 7, 3, 8
    g = RNG.standard_normal((5, T, H, D))
    w = RNG.standard_normal((H, D, D, 5))
    out = O.conv_compress(g, w)
    for h in range(H):
        inp = torch.from_numpy(np.ascontiguousarray(g[:, :, h, :].transpose(1, 2, 0)))  # [T, D_in, 5]
        ref = torch.nn.functional.conv1d(inp, torch.from_numpy(w[h]), stride=5)          # [T, D_out, 1]
        np.testing.assert_allclose(out[:, h, :], ref[:, :, 0].numpy(), rtol=1e-13, atol=1e-13)


def test_conv_mean_pool_closed_form():
    g = RNG.standard_normal((5, 6, 2, 4))
    w = np.zeros((2, 4, 4, 5))
    for o in range(4):
        w[:, o, o, :] = 0.2
    np.testing.assert_allclose(O.conv_compress(g, w), g.mean(axis=0), atol=1e-15)


def test_conv_constant_weight_closed_form():
    g = RNG.standard_normal((5, 6, 2, 4))
    w = np.full((2, 4, 4, 5), 0.37)
    ref = 0.37 * g.sum(axis=(0, 3))
    out = O.conv_compress(g, w)
    for o in range(4):
        np.testing.assert_allclose(out[:, :, o], ref, atol=1e-13)


def test_conv_single_entry_orientation():
    # only w[h=1, o=2, i=3, j=4] = 1: output channel 2 of head 1 copies input channel 3 of the
    # newest (5th) frame; every other output is 0 (catches o/i and tap-order transpositions)
    g = RNG.standard_normal((5, 6, 2, 4))
    w = np.zeros((2, 4, 4, 5)); w[1, 2, 3, 4] = 1.0
    out = O.conv_compress(g, w)
    np.testing.assert_array_equal(out[:, 1, 2], g[4, :, 1, 3])
    mask = np.ones_like(out, dtype=bool); mask[:, 1, 2] = False
    assert np.all(out[mask] == 0)


# ---------------------------------------------------------------- attention

def test_attention_matches_torch_sdpa():
    q = RNG.standard_normal((9, 64)); k = RNG.standard_normal((40, 64)); v = RNG.standard_normal((40, 64))
    o, ps = O.attend_rows(q, k, v)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])[0].numpy()
    np.testing.assert_allclose(o, ref, atol=1e-13)
    np.testing.assert_allclose(ps, 1.0, atol=1e-12)


def test_attention_single_key_and_zero_keys():
    q = RNG.standard_normal((3, 8)); k = RNG.standard_normal((1, 8)); v = RNG.standard_normal((1, 8))
    np.testing.assert_allclose(O.attend_rows(q, k, v)[0], np.repeat(v, 3, 0), atol=1e-15)
    # K = 0: uniform weights, output = mean of V
    k0 = np.zeros((17, 8)); v = RNG.standard_normal((17, 8))
    np.testing.assert_allclose(O.attend_rows(q, k0, v)[0], np.repeat(v.mean(0, keepdims=True), 3, 0), atol=1e-14)


def test_attention_two_key_logistic_form():
    # two keys: weight of key 0 is the logistic function of the score difference
    q = RNG.standard_normal((4, 16)); k = RNG.standard_normal((2, 16)); v = np.eye(2, 16)
    o, _ = O.attend_rows(q, k, v)
    d = (q @ (k[0] - k[1])) / 4.0
    np.testing.assert_allclose(o[:, 0], 1.0 / (1.0 + np.exp(-d)), atol=1e-14)


def test_attention_key_permutation_invariance():
    q = RNG.standard_normal((5, 32)); k = RNG.standard_normal((50, 32)); v = RNG.standard_normal((50, 32))
    perm = RNG.permutation(50)
    np.testing.assert_allclose(O.attend_rows(q, k, v)[0], O.attend_rows(q, k[perm], v[perm])[0], atol=1e-14)


# ---------------------------------------------------------------- stream bookkeeping

def _tiny_stream(W, C, blocks, b=2, b1=None, fp8=False, H=2, D=64, gh=4, gw=4, seed=0, fp4=False):
    cfg = O.OracleConfig(H=H, D=D, grid_h=gh, grid_w=gw, window=W, mem_slots=C, fp8=fp8, fp4=fp4)
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((2, H, D, D, 5)) / math.sqrt(5 * D)
    st = O.OracleStream(cfg, w)
    data = []
    for n in range(blocks):
        bb = (b1 if (b1 and n == 0) else b)
        k = rng.standard_normal((bb, cfg.T, H, D)); v = rng.standard_normal((bb, cfg.T, H, D))
        q = rng.standard_normal((bb, cfg.T, H, D))
        st.append(k, v)
        data.append((q, k, v))
        yield st, (q, k, v), data


def _read_golden():
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_stream_layout.txt")
    rows = []
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        f = line.split()
        rows.append(f)
    return rows


def _frames(spec):
    if spec == "-":
        return []
    out = []
    for part in spec.split(","):
        if "-" in part:
            a, b = part.split("-"); out += list(range(int(a), int(b) + 1))
        else:
            out.append(int(part))
    return out


def test_tiny_stream_matches_hand_table():
    gold = _read_golden()
    cfg = O.OracleConfig(H=1, D=6, grid_h=1, grid_w=1, window=4, mem_slots=3)
    st = O.OracleStream(cfg, np.zeros((2, 1, 6, 6, 5)))
    for row in gold:
        blk, m, w = int(row[0]), int(row[1]), int(row[2])
        ev = st.append(np.zeros((2, 1, 1, 6)), np.zeros((2, 1, 1, 6)))
        assert st.block == blk and (st.m, st.w_frames) == (m, w), row
        assert [e.first_frame for e in ev] == _frames(row[3])
        assert [5 * f.index for f in st.memory] == _frames(row[4])
        assert [f.index for f in st.window] == _frames(row[5])
        assert [f.index for f in st.current] == _frames(row[6])
        lay = st.layout()
        # time indices restart at 0 and run over memory, window, current in order
        assert list(lay[:, 2]) == list(range(len(lay)))


def _closed_form(P, W, C):
    """Closed form of the counters after promoting P frames in total."""
    E = 5 * math.ceil(max(0, P - W) / 5)
    S = E // 5
    return E, P - E, S, min(S, C)


@pytest.mark.parametrize("b1,b,W,C,frames", [(6, 8, 10, 8, 18000), (6, 8, 10, 16, 300), (8, 8, 10, 8, 200),
                                             (2, 2, 4, 3, 30)])
def test_bookkeeping_closed_form(b1, b, W, C, frames):
    cfg = O.OracleConfig(H=1, D=6, grid_h=1, grid_w=1, window=W, mem_slots=C)
    st = O.OracleStream(cfg, np.zeros((2, 1, 6, 6, 5)))
    sizes = [b1] + [b] * ((frames - b1) // b)
    if sum(sizes) < frames:
        sizes.append(frames - sum(sizes))
    z = {n: np.zeros((n, 1, 1, 6)) for n in set(sizes)}
    total = 0
    max_items = 0
    for n in sizes:
        st.append(z[n], z[n])
        E, w, S, m = _closed_form(total, W, C)
        assert (st.E, st.w_frames, st.S, st.m) == (E, w, S, m)
        # stored slots are S-m .. S-1, slot k covers frames [5k, 5k+5)
        assert [f.index for f in st.memory] == list(range(S - m, S))
        assert [f.index for f in st.window] == list(range(E, total))
        total += n
        max_items = max(max_items, st.m + st.w_frames + len(st.current))
    # constant footprint: stored items never exceed C + W + max block
    assert max_items <= C + W + max(b1, b)


def test_first_conv_at_third_block_512_config():
    # blocks of 6 then 8, W = 10: the first compression runs at the third block, as the
    # Streaming Pipeline section states (blocks 1-2 uncompressed, ConvKV from block 3)
    cfg = O.OracleConfig(H=1, D=6, grid_h=1, grid_w=1, window=10, mem_slots=8)
    st = O.OracleStream(cfg, np.zeros((2, 1, 6, 6, 5)))
    st.append(np.zeros((6, 1, 1, 6)), np.zeros((6, 1, 1, 6)))
    st.append(np.zeros((8, 1, 1, 6)), np.zeros((8, 1, 1, 6)))
    assert st.events == []
    ev = st.append(np.zeros((8, 1, 1, 6)), np.zeros((8, 1, 1, 6)))
    assert [(e.block, e.first_frame, e.slot) for e in ev] == [(3, 0, 0)]


# ---------------------------------------------------------------- stream attention

def test_stream_without_eviction_equals_full_attention():
    """W larger than the stream: no eviction, m = 0, so reset positions equal absolute frame
    indices and the step is block-causal full attention over frames [0, end of block n]."""
    H, D, gh, gw = 2, 64, 4, 4
    T = gh * gw
    ks, vs = [], []
    for st, (q, k, v), _ in _tiny_stream(W=100, C=3, blocks=5, H=H, D=D, gh=gh, gw=gw, seed=5):
        ks.append(k); vs.append(v)
        o, ps = st.attend(q)
        kall = np.concatenate(ks).reshape(-1, H, D); vall = np.concatenate(vs).reshape(-1, H, D)
        nk = kall.shape[0]
        f_k = np.arange(nk) // T; s_k = np.arange(nk) % T
        f_q = (nk - q.shape[0] * T) // T + np.arange(q.shape[0] * T) // T
        s_q = np.arange(q.shape[0] * T) % T
        qq = q.reshape(-1, H, D)
        for h in range(H):
            kr = _rope_complex(kall[:, h], f_k, s_k // gw, s_k % gw, (24, 20, 20), 1e4)
            qr = _rope_complex(qq[:, h], f_q, s_q // gw, s_q % gw, (24, 20, 20), 1e4)
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(qr)[None], torch.from_numpy(kr)[None], torch.from_numpy(vall[:, h])[None])[0]
            np.testing.assert_allclose(o[:, h], ref.numpy(), atol=1e-12)
        np.testing.assert_allclose(ps, 1.0, atol=1e-12)


def test_stream_uniform_time_shift_invariance():
    for st, (q, k, v), _ in _tiny_stream(W=4, C=3, blocks=12, seed=7):
        pass
    rows = np.arange(0, 32, 3)
    o0, _ = st.attend(q, rows=rows)
    o1, _ = st.attend(q, rows=rows, t_offset=1000)
    np.testing.assert_allclose(o0, o1, atol=1e-12)


def test_stream_key_order_invariance():
    """Shuffling the key frames with their positions attached leaves the output unchanged."""
    for st, (q, k, v), _ in _tiny_stream(W=4, C=3, blocks=9, seed=9):
        pass
    rows = np.arange(0, 32, 5)
    o0, _ = st.attend(q, rows=rows)
    kf = st.key_frames()
    st2_memory, st2_window = list(st.memory), list(st.window)
    # reverse the memory FIFO but keep each slot's own time index by overriding key_frames
    perm = list(reversed(kf))
    st.key_frames = lambda: perm
    o1, _ = st.attend(q, rows=rows)
    np.testing.assert_allclose(o0, o1, atol=1e-12)


def test_stream_memory_slots_are_bf16_conv_of_group():
    gen = _tiny_stream(W=4, C=3, blocks=4, seed=11)
    hist = []
    for st, (q, k, v), _ in gen:
        hist.append((k, v))
    frames_k = np.concatenate([h[0] for h in hist])
    kc, vc = st.memory_slot(0)
    ref = O.round_to_bf16(O.conv_compress(frames_k[0:5], st.w[0]))
    np.testing.assert_array_equal(kc, ref)
    # every stored value is a bf16 value
    np.testing.assert_array_equal(O.round_to_bf16(vc), vc)


def test_fp8_stream_window_is_quantised_current_is_exact():
    for st, (q, k, v), _ in _tiny_stream(W=4, C=3, blocks=5, fp8=True, seed=13):
        pass
    # current block frames are the exact inputs; window frames are per-(head, frame) e4m3
    # codes (fixed points of the quantiser) dequantised to bf16
    np.testing.assert_array_equal(st.current[0].k, k[0])
    for f in st.window:
        ck, sk, cv, sv = f.codes
        np.testing.assert_array_equal(O.e4m3_rne_satfinite(ck.astype(np.float32)), ck)
        np.testing.assert_array_equal(sk, st.frame_scales[f.index][0])
        np.testing.assert_array_equal(f.k, O.fp8_dequantize(ck, sk))
        np.testing.assert_array_equal(O.round_to_bf16(f.k), f.k)


def test_sink_partition_equals_full_attention_over_concatenated_keys():
    """With a reference-image partition, the output is the attention over
    [sink | memory | window | current] with positions 0.. in that order: the same
    as a stream without sink whose keys are prefixed by the sink frames and whose
    time indices (queries included) are shifted by the sink length."""
    H, D, gh, gw = 2, 64, 4, 4
    T = gh * gw
    rng = np.random.default_rng(21)
    cfg = O.OracleConfig(H=H, D=D, grid_h=gh, grid_w=gw, window=4, mem_slots=3)
    w = rng.standard_normal((2, H, D, D, 5)) / 16
    st = O.OracleStream(cfg, w)
    sk, sv = rng.standard_normal((2, T, H, D)), rng.standard_normal((2, T, H, D))
    st.set_sink(sk, sv)
    for n in range(7):
        k, v, q = (rng.standard_normal((2, T, H, D)) for _ in range(3))
        st.append(k, v)
    o, ps = st.attend(q)
    np.testing.assert_allclose(ps, 1.0, atol=1e-12)
    lay = st.layout()
    assert list(lay[:2, 0]) == [O.PART_SINK] * 2 and list(lay[:, 2]) == list(range(len(lay)))
    # independent restatement: rotate with the complex form, SDPA over all key frames
    kf = st.key_frames()
    tok = np.arange(T)
    for h in range(H):
        kall = np.concatenate([f.k[:, h, :] for _, f, _ in kf])
        vall = np.concatenate([f.v[:, h, :] for _, f, _ in kf])
        kt = np.concatenate([np.full(T, t) for _, _, t in kf])
        kr = _rope_complex(kall, kt, np.tile(tok // gw, len(kf)), np.tile(tok % gw, len(kf)), (24, 20, 20), 1e4)
        qq = q[:, :, h, :].reshape(-1, D)
        qt = len(kf) - 2 + np.arange(2 * T) // T
        qr = _rope_complex(qq, qt, np.tile(tok // gw, 2), np.tile(tok % gw, 2), (24, 20, 20), 1e4)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qr)[None], torch.from_numpy(kr)[None], torch.from_numpy(vall)[None])[0].numpy()
        np.testing.assert_allclose(o[:, h], ref, atol=1e-12)


# -- NVFP4 (e2m1 values, e4m3 block scales per 16 channels, fp32 scale per frame and head)

def test_e2m1_hand_table():
    """The e2m1 grid {0, .5, 1, 1.5, 2, 3, 4, 6}: nearest value, ties to the even
    mantissa, saturation at 6 (values written out by hand from the format)."""
    x = [0.0, 0.1, 0.25, 0.2500001, 0.5, 0.74, 0.75, 0.76, 1.0, 1.24, 1.25, 1.26, 1.5, 1.75, 2.0,
         2.49, 2.5, 2.51, 3.0, 3.5, 4.0, 4.99, 5.0, 5.01, 6.0, 7.0, 100.0, -0.75, -5.0, -7.0, -0.25]
    want = [0.0, 0.0, 0.0, 0.5, 0.5, 0.5, 1.0, 1.0, 1.0, 1.0, 1.0, 1.5, 1.5, 2.0, 2.0,
            2.0, 2.0, 3.0, 3.0, 4.0, 4.0, 4.0, 4.0, 6.0, 6.0, 6.0, 6.0, -1.0, -4.0, -6.0, -0.0]
    got = O.e2m1_rne_satfinite(np.array(x, dtype=np.float32))
    np.testing.assert_array_equal(got, np.array(want))


def test_e2m1_matches_brute_force_nearest():
    """Against a search over the 15 finite values: nearest, and on a tie the one whose
    mantissa bit is 0 (code index even)."""
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.uniform(-8, 8, 20000), (np.arange(-16, 17) / 4.0)]).astype(np.float32)
    ref = np.empty(len(x))
    for i, v in enumerate(x.astype(np.float64)):
        a = min(abs(v), 6.0)
        d = np.abs(mags - a)
        best = np.flatnonzero(d == d.min())
        j = best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]
        ref[i] = math.copysign(mags[j], v) if mags[j] != 0 else 0.0
    np.testing.assert_array_equal(np.abs(O.e2m1_rne_satfinite(x)), np.abs(ref))


def test_fp4_encode_grid_values_round_trip():
    """Hand example.  Block 0 holds e2m1 grid values with max 6 = the frame's amax:
    g = fp32(6 / 2688), s_0 = e4m3(6 / fp32(6 g)) = 448, e_0 = fp32(448 g) = 1, so the
    codes are the values themselves.  Block 1 holds half-grid values with max 3:
    s_1 = e4m3(3 / fp32(6 g)) = 224, e_1 = 1/2, codes = 2x.  Both dequantise exactly."""
    b0 = [6.0, -3.0, 1.5, 0.5, 0.0, 4.0, -6.0, 2.0, 1.0, -1.5, 3.0, -0.5, 0.0, -4.0, 2.0, 1.0]
    b1 = [v / 2 for v in b0]
    x = np.array(b0 + b1, dtype=np.float64).reshape(1, 1, 32)
    code, sb, g = O.fp4_encode(x)
    assert g.dtype == np.float32 and g[0] == np.float32(6.0) / np.float32(2688.0)
    np.testing.assert_array_equal(sb[0, 0], [448.0, 224.0])
    np.testing.assert_array_equal(code[0, 0, :16], b0)
    np.testing.assert_array_equal(code[0, 0, 16:], [2 * v for v in b1])
    np.testing.assert_array_equal(O.fp4_dequantize(code, sb, g), x)


def test_fp4_zero_block_and_error_bound():
    rng = np.random.default_rng(9)
    x = O.round_to_bf16(rng.standard_normal((8, 3, 64)))
    x[2, 1, 16:32] = 0.0                                   # an all-zero block
    code, sb, g = O.fp4_encode(x)
    assert sb[2, 1, 1] == 0 and np.all(code[2, 1, 16:32] == 0)
    np.testing.assert_array_equal(O.e2m1_rne_satfinite(code.astype(np.float32)), code)   # codes on the grid
    np.testing.assert_array_equal(O.e4m3_rne_satfinite(sb.astype(np.float32)), sb)      # scales on the grid
    dq = O.fp4_dequantize(code, sb, g)
    eb = (sb * g[None, :, None]).repeat(16, axis=2)
    # |x/e - code| <= 1 (largest half-quantum, at |x/e| in [4, 6]) plus the bf16 rounding
    assert np.all(np.abs(dq - x) <= eb * 1.0 + np.abs(x) * 2.0 ** -8 + 1e-30)


def test_fp4_stream_window_is_quantised_current_is_exact():
    for st, (q, k, v), _ in _tiny_stream(W=4, C=3, blocks=5, fp4=True, seed=17):
        pass
    np.testing.assert_array_equal(st.current[0].k, k[0])
    assert len(st.memory) > 0 and len(st.window) > 0
    for f in st.window + st.memory:
        ck, (bk, gk), cv, (bv, gv) = f.codes
        np.testing.assert_array_equal(O.e2m1_rne_satfinite(ck.astype(np.float32)), ck)
        np.testing.assert_array_equal(f.k, O.fp4_dequantize(ck, bk, gk))
        np.testing.assert_array_equal(f.v, O.fp4_dequantize(cv, bv, gv))
    o, ps = st.attend(q)
    np.testing.assert_allclose(ps, 1.0, atol=1e-12)


@pytest.mark.parametrize("fmt", ["fp8", "fp4"])
def test_low_precision_memory_slot_is_encoded_conv_of_dequantised_group(fmt):
    """A stored memory slot in the low-precision formats is the conv of its group's five
    frames as the cache holds them (each quantised when it joined the window, then
    dequantised to BF16 on use), encoded once more in the cache's format: slot k covers
    stream frames [5k, 5k+5).  Codes and scales must match that composition exactly, and
    the slot's values must be their dequantisation (model card, --fp8_kv_cache: stored
    in FP8, dequantised to BF16 on use)."""
    fp4 = fmt == "fp4"
    enc = (lambda x: (lambda c, sb, g: (c, (sb, g)))(*O.fp4_encode(x))) if fp4 else O.fp8_encode
    deq = (lambda c, s: O.fp4_dequantize(c, s[0], s[1])) if fp4 else O.fp8_dequantize
    hist = []
    for st, (q, k, v), _ in _tiny_stream(W=4, C=3, blocks=12, fp8=not fp4, fp4=fp4, seed=29):
        hist.append((k, v))
    K = np.concatenate([h[0] for h in hist])
    V = np.concatenate([h[1] for h in hist])
    assert st.S > st.m == 3          # the FIFO has dropped slots
    for age, slot in enumerate(st.memory):
        f0 = 5 * slot.index
        for kv, (X, got_val, got_codes) in enumerate(((K, slot.k, slot.codes[:2]), (V, slot.v, slot.codes[2:]))):
            group = np.stack([deq(*enc(X[f])) for f in range(f0, f0 + 5)])
            code, scales = enc(O.conv_compress(group, st.w[kv]))
            np.testing.assert_array_equal(got_codes[0], code)
            if fp4:
                np.testing.assert_array_equal(got_codes[1][0], scales[0])
                np.testing.assert_array_equal(got_codes[1][1], scales[1])
            else:
                np.testing.assert_array_equal(got_codes[1], scales)
            np.testing.assert_array_equal(got_val, deq(code, scales))

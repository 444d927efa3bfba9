"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Every check compares the library's result with the oracle on the same seeded
inputs.  Indices (layout, slot positions) must be bit-exact, appended ring
frames must be bit-exact copies, attention outputs and compressed slots must
hold the stated tolerances.
"""
import numpy as np
import pytest

import seeded_inputs as si
from compressed_kv_cache_convkv_b200.configs import PRESETS, Workload
from dataclasses import replace

from streams import (attention_errors, bf16_tensor_to_f64, check_attention, check_codes, check_codes_fp4, check_slot,
                     device_frames, device_weights, host_frames, oracle_for, sample_rows, select_heads,
                     check_attention_scaled)

# NVFP4 conv outputs: fraction of channels allowed to sit one step apart (a code or its
# block scale next to a rounding boundary; 8e-6 at most on the 480x832 stream)
FP4_VALUE_MISMATCH = 1e-4

pytestmark = pytest.mark.gpu

# Heads the oracle evaluates at the 40-head shapes.  Heads are independent through the
# whole step (per-head conv weights, per-head quantisation scales, per-head attention),
# so the oracle run on a head subset gives exactly those heads' values; the subsets
# include the first and the last head and spread over the rest.
HEADS8 = (0, 5, 11, 17, 22, 28, 33, 39)


@pytest.fixture(scope="module")
def torch():
    import torch as t
    assert t.cuda.is_available(), "GPU tests need a CUDA device"
    from compressed_kv_cache_convkv_b200 import build
    build.build()
    si.build(device=True)
    return t


def _ckv():
    import compressed_kv_cache_convkv_b200 as ckv
    return ckv


def test_device_generator_matches_host(torch):
    w = PRESETS["720x416"]
    d = device_frames(w, si.K, 7, 2, torch)[0]
    h = host_frames(w, si.K, 0, 7, 2).reshape(-1, w.heads, w.head_dim)
    assert np.array_equal(d.view(torch.int16).cpu().numpy().view(np.uint16), h)


def test_bounded_wait_reports_timeout_and_context_survives(torch):
    """A kernel whose barrier never completes gives up after its budget (~10 ms here),
    reports CONVKV_ERR_DEVICE_TIMEOUT through the status word, and the context keeps
    working (the tiny stream still matches the oracle afterwards)."""
    import time
    ckv = _ckv()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    rc = ckv.library().convkv_selftest_wait_timeout(status.data_ptr(), 20_000_000,
                                                    torch.cuda.current_stream().cuda_stream)
    assert rc == ckv.ERR_DEVICE_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert int(status.item()) != 0
    assert ckv.library().convkv_selftest_wait_timeout(status.data_ptr(), 10, 0) == ckv.ERR_INVALID_ARG
    _run(torch, PRESETS["tiny"], max_blocks=5)


def test_quantiser_division_matches_ieee(torch):
    """The e4m3 / NVFP4 quantisers' shared-divisor quotient (two Markstein correction
    steps after RN(x * RN(1/s))) equals CUDA's IEEE fp32 division bit for bit: random
    pairs over the quantisers' ranges, divisors outside the fast path's range, zeros,
    and quotients placed next to fp32 rounding midpoints."""
    ckv = _ckv()
    g = torch.Generator(device="cuda").manual_seed(11)
    n = 1 << 23
    dev = "cuda"

    def rand(*shape, dtype=torch.float32):
        return torch.rand(*shape, device=dev, generator=g, dtype=dtype)

    def randint(lo, hi):
        return torch.randint(lo, hi, (n,), device=dev, generator=g)

    sets = []
    # quotients up to 448 in magnitude over divisors 2^-70 .. 2^60 (below 2^-60: IEEE path)
    s = ((rand(n) + 1) * torch.exp2(randint(-70, 60).float())).float()
    x = ((rand(n, dtype=torch.float64) * 896 - 448) * s.double()).float()
    sets.append((x, s))
    # quotients within a few 2^-25 units of the last place of an fp32 rounding midpoint
    m = randint(2 ** 23, 2 ** 24).double()
    e = randint(-11, 9).double()
    k = randint(-4, 5).double()
    mid = (m + 0.5 + k * 2.0 ** -25) * torch.exp2(e - 23)
    s = ((rand(n) + 1) * torch.exp2(randint(-40, 30).float())).float()
    sets.append(((mid * s.double()).float(), s))
    # arbitrary dividends, bf16-grid dividends, zeros of both signs
    s = ((rand(n) + 1) * torch.exp2(randint(-20, 20).float())).float()
    x = (torch.randn(n, device=dev, generator=g) * torch.exp2(randint(-30, 30).float())).bfloat16().float()
    x[: n // 64] = 0.0
    x[n // 64: n // 32] = -0.0
    sets.append((x, s))
    bad = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    for xs, ss in sets:
        xs, ss = xs.contiguous(), ss.contiguous()
        assert bool(torch.isfinite(xs).all()) and bool((ss > 0).all())
        assert ckv.library().convkv_selftest_div_rn(xs.data_ptr(), ss.data_ptr(), n, bad.data_ptr(), stream) == 0
    assert int(bad.item()) == 0


def _run(torch, w: Workload, attend_blocks=None, rows=None, compress=0, t_offset=0, override=None,
         check_slots=True, ring_frames=None, max_blocks=None, collect=None, sharp=False, sink=0, heads=None):
    """Stream w through both sides; returns per-block error records.  sink > 0 gives both
    sides that many reference-image frames (attended first, never evicted).  heads: the
    heads the oracle evaluates and the checks compare (all when None)."""
    ckv = _ckv()
    weights = device_weights(w, torch)
    cfg = w.config(compress_mode=compress, t_offset=t_offset, sink_frames=sink)
    h = ckv.ConvKV(cfg, None if compress == ckv.COMPRESS_MEAN else weights)
    st = oracle_for(w, mean=(compress == ckv.COMPRESS_MEAN), heads=heads)
    if sink:
        _set_sink(torch, w, h, {0: st}, sink, heads)
    rng = np.random.default_rng(w.seed)
    R = cfg.ring_frames
    F = 0
    recs = []
    sizes = w.block_sizes()[: max_blocks or None]
    for n, b in enumerate(sizes, start=1):
        kd, vd, qd = (device_frames(w, t, F, b, torch) for t in (si.K, si.V, si.Q))
        kh, vh, qh = (host_frames(w, t, 0, F, b, heads) for t in (si.K, si.V, si.Q))
        if override is not None:
            kd, vd, qd, kh, vh, qh = override(torch, kd, vd, qd, kh, vh, qh)
        h.append(kd, vd)
        out = h.attend(qd)
        ev = st.append(si.bf16_bits_to_f64(kh), si.bf16_bits_to_f64(vh))
        # indices: bit-exact layout
        lay = h.layout()
        assert [tuple(r) for r in lay[:, [0, 1, 3]]] == [tuple(r) for r in st.layout()], f"block {n}"
        c = h.counters()
        assert (c["P"], c["E"], c["S"], c["groups"]) == (st.P, st.E, st.S, len(ev))
        # append: ring frames are bit-exact copies of the inputs
        frames = range(b) if ring_frames is None else [x for x in ring_frames if x < b]
        for f in frames:
            kb, _ = h.read_ring(0, 0, (F + f) % R)
            vb, _ = h.read_ring(0, 1, (F + f) % R)
            kb, vb = select_heads(kb, heads), select_heads(vb, heads)
            assert np.array_equal(kb, kh[f]) and np.array_equal(vb, vh[f]), f"ring frame {F + f}"
        # compression: new memory slots
        if check_slots:
            for e in ev[-cfg.mem_slots:]:
                pos = e.slot % cfg.mem_slots
                age = st.m - (st.S - e.slot)
                ref_k, ref_v = st.memory_slot(age)
                gk, _ = h.read_slot(0, 0, pos)
                gv, _ = h.read_slot(0, 1, pos)
                gk, gv = select_heads(gk, heads), select_heads(gv, heads)
                ek = check_slot(si.bf16_bits_to_f64(gk), ref_k, f"K slot {e.slot}")
                ev_ = check_slot(si.bf16_bits_to_f64(gv), ref_v, f"V slot {e.slot}")
                recs.append(("slot", n, e.slot, ek, ev_))
        # attention
        if attend_blocks is None or n in attend_blocks:
            r = sample_rows(w, b, rows or b * w.T, rng)
            ref, psum = st.attend(si.bf16_bits_to_f64(qh), rows=r)
            assert np.abs(psum - 1).max() < 1e-12
            gpu = select_heads(bf16_tensor_to_f64(out[0][torch.as_tensor(r, device="cuda")]), heads)
            e = check_attention(gpu, ref, what=f"{w.name} block {n}", sharp=sharp)
            recs.append(("attend", n, len(r), e))
            if collect is not None:
                collect.append((n, r, gpu, ref))
        F += b
    assert h.status() == 0
    h.close()
    return recs


def _set_sink(torch, w, h, oracles, sink, heads=None):
    """heads: None, one head subset for every oracle, or a dict state -> subset."""
    h.set_sink(device_frames(w, si.RK, 0, sink, torch), device_frames(w, si.RV, 0, sink, torch))
    for s, st in oracles.items():
        hs = heads.get(s) if isinstance(heads, dict) else heads
        st.set_sink(si.bf16_bits_to_f64(host_frames(w, si.RK, s, 0, sink, hs)),
                    si.bf16_bits_to_f64(host_frames(w, si.RV, s, 0, sink, hs)))


def test_tiny_stream_full_parity(torch):
    recs = _run(torch, PRESETS["tiny"])
    assert sum(1 for r in recs if r[0] == "slot") == 5        # conv events at blocks 4, 6, 9, 11, 14
    assert sum(1 for r in recs if r[0] == "attend") == 15


def test_tiny_mean_memory(torch):
    ckv = _ckv()
    _run(torch, PRESETS["tiny"], compress=ckv.COMPRESS_MEAN)


def test_512_mean_memory(torch):
    """The 5-frame mean in place of the conv at the production head size (D=128, 40 heads)."""
    ckv = _ckv()
    _run(torch, PRESETS["512x512"], compress=ckv.COMPRESS_MEAN, attend_blocks={3, 7, 13, 26}, rows=128,
         ring_frames=[0], heads=HEADS8)


def test_tiny_time_shift_invariance(torch):
    """Adding 1000 to every RoPE time index changes nothing (RoPE is relative)."""
    a, b = [], []
    _run(torch, PRESETS["tiny"], t_offset=0, collect=a)
    _run(torch, PRESETS["tiny"], t_offset=1000, collect=b)
    for (n, r, g0, ref), (_, _, g1, _) in zip(a, b):
        e = attention_errors(g1, g0)
        assert e["max"] <= 1e-2 and e["rel_l2"] <= 1e-2, (n, e)


def test_tiny_v_ones_gives_ones(torch):
    """V = 1 everywhere and mean compression: every output is 1 up to the bf16 rounding
    of the attention weights (each weight is rounded to bf16 for the PV product, relative
    error <= 2^-8, while the row sum uses the unrounded weights)."""
    ckv = _ckv()

    def ones_v(t, kd, vd, qd, kh, vh, qh):
        vd = t.ones_like(vd)
        vh = np.full_like(vh, 0x3F80)
        return kd, vd, qd, kh, vh, qh

    col = []
    _run(torch, PRESETS["tiny"], compress=ckv.COMPRESS_MEAN, override=ones_v, collect=col)
    for n, r, gpu, ref in col:
        assert np.abs(gpu - 1.0).max() <= 2.0 ** -8, n
        assert np.mean(gpu == 1.0) > 0.9, n


def test_tiny_k_zero_gives_mean_of_valid_v(torch):
    """K = 0: uniform weights, so a padded key leaking into a ragged tile would show."""
    def zero_k(t, kd, vd, qd, kh, vh, qh):
        return t.zeros_like(kd), vd, qd, np.zeros_like(kh), vh, qh

    _run(torch, PRESETS["tiny"], override=zero_k)


def test_tiny_sharp_softmax(torch):
    """Queries scaled by 8: peaky softmax exercises the running-max rescale."""
    def sharp(t, kd, vd, qd, kh, vh, qh):
        qd = (qd.float() * 8).to(t.bfloat16)
        qh8 = si.bf16_bits_to_f64(qh) * 8
        qh = (qh8.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
        return kd, vd, qd, kh, vh, qh

    _run(torch, PRESETS["tiny"], override=sharp, sharp=True)


def test_512_stream(torch):
    _run(torch, PRESETS["512x512"], attend_blocks={1, 3, 4, 7, 9, 13, 20, 26}, rows=256, ring_frames=[0, 5],
         heads=HEADS8)


def test_720_stream_ragged(torch):
    _run(torch, PRESETS["720x416"], attend_blocks={1, 3, 12, 13, 27, 38}, rows=256, ring_frames=[0, 5],
         heads=HEADS8)


def _run_fp8(torch, w: Workload, states=(0,), attend_blocks=None, rows=None, ring_frames=None, sink=0,
             heads=None, outliers=False, max_blocks=None):
    """Low-precision formats (e4m3, or NVFP4 when w.fp4): window codes and scales bit-exact,
    memory codes within one step, attention <= 5e-2.  heads: dict state -> the heads the
    oracle evaluates for that state (all when None).  outliers: K and V carry a few
    x16 values per frame and head (heavy tails beyond the unit-variance inputs)."""
    ckv = _ckv()
    weights = device_weights(w, torch)
    cfg = w.config(sink_frames=sink)
    h = ckv.ConvKV(cfg, weights)
    hsel = lambda s: None if heads is None else heads[s]
    oracles = {s: oracle_for(w, state=s, heads=hsel(s)) for s in states}
    if sink:
        _set_sink(torch, w, h, oracles, sink, heads)
    rng = np.random.default_rng(w.seed)
    R = cfg.ring_frames
    F = 0
    for n, b in enumerate(w.block_sizes()[: max_blocks or None], start=1):
        kd, vd, qd = (device_frames(w, t, F, b, torch) for t in (si.K, si.V, si.Q))
        host = {}
        for s in states:
            host[s] = [host_frames(w, t, s, F, b, hsel(s)) for t in (si.K, si.V, si.Q)]
        if outliers:
            pos = _outlier_positions(w, F, b)
            for x in (kd, vd):
                _scale_device(torch, w, x, pos)
            for s in states:
                for i in (0, 1):
                    host[s][i] = _scale_host(w, host[s][i], pos, hsel(s))
        h.append(kd, vd)
        out = h.attend(qd)
        for s, st in oracles.items():
            hs = hsel(s)
            kh, vh, qh = host.pop(s)
            ev = st.append(si.bf16_bits_to_f64(kh), si.bf16_bits_to_f64(vh))
            del kh, vh
            if s == states[0]:
                lay = h.layout()
                assert [tuple(r) for r in lay[:, [0, 1, 3]]] == [tuple(r) for r in st.layout()], f"block {n}"
                assert [int(x) for x in lay[lay[:, 0] == 2, 2]] == list(range(b))  # staging slots
            # the new block's ring codes and scales: bit-exact
            frames = range(b) if ring_frames is None else [x for x in ring_frames if x < b]
            for f in frames:
                ck, sk, cv, sv = st.current_q8[f].codes
                for kv, (rc, rsc) in enumerate(((ck, sk), (cv, sv))):
                    gb, gs = _sel_q(h.read_ring(s, kv, (F + f) % R), hs, w.fp4)
                    what = f"state {s} frame {F + f} kv {kv}"
                    if w.fp4:
                        check_codes_fp4((gb, gs), (rc, rsc), exact=True, what=what)
                    else:
                        check_codes(gb, gs, rc, rsc, exact=True, what=what)
            # new memory slots: codes within one step of the oracle's
            for e in ev[-cfg.mem_slots:]:
                age = st.m - (st.S - e.slot)
                ck, sk, cv, sv = st.memory[age].codes
                for kv, (rc, rsc) in enumerate(((ck, sk), (cv, sv))):
                    gb, gs = _sel_q(h.read_slot(s, kv, e.slot % cfg.mem_slots), hs, w.fp4)
                    what = f"state {s} slot {e.slot} kv {kv}"
                    if w.fp4:
                        check_codes_fp4((gb, gs), (rc, rsc), exact=False, what=what, max_frac=FP4_VALUE_MISMATCH)
                    else:
                        check_codes(gb, gs, rc, rsc, exact=False, what=what)
            if attend_blocks is None or n in attend_blocks:
                r = sample_rows(w, b, rows or b * w.T, rng)
                ref, _ = st.attend(si.bf16_bits_to_f64(qh), rows=r)
                gpu = select_heads(bf16_tensor_to_f64(out[s][torch.as_tensor(r, device="cuda")]), hs)
                if outliers:
                    check_attention_scaled(gpu, ref, what=f"{w.name} outliers state {s} block {n}")
                else:
                    check_attention(gpu, ref, fp8=True, what=f"{w.name} state {s} block {n}")
        F += b
    assert h.status() == 0
    h.close()


# -- heavy-tailed inputs -------------------------------------------------------

OUTLIERS_PER_FRAME_HEAD, OUTLIER_GAIN = 4, 16.0


def _outlier_positions(w, F, b):
    """(block frame, token, head, channel) of the x16 values: 4 per frame and head, at
    positions that move with the stream frame and the head."""
    T, H, D = w.T, w.heads, w.head_dim
    pos = []
    for f in range(b):
        g = F + f
        for h in range(H):
            for i in range(OUTLIERS_PER_FRAME_HEAD):
                tok = (g * 31 + h * 17 + i * (T // OUTLIERS_PER_FRAME_HEAD) + 5) % T
                ch = (g * 7 + h * 3 + i * 29) % D
                pos.append((f, tok, h, ch))
    return np.array(pos, dtype=np.int64)


def _scale_device(torch, w, x, pos):
    """x16 at `pos` in every state of the device block x[S, b*T, H, D] (exact in bf16)."""
    rows = torch.as_tensor(pos[:, 0] * w.T + pos[:, 1], device="cuda")
    hh = torch.as_tensor(pos[:, 2], device="cuda")
    cc = torch.as_tensor(pos[:, 3], device="cuda")
    x[:, rows, hh, cc] = x[:, rows, hh, cc] * OUTLIER_GAIN


def _scale_host(w, bits, pos, heads):
    """The same on the host bits [b, T, H', D] of the heads in `heads` (all when None)."""
    vals = si.bf16_bits_to_f64(bits)
    hmap = {h: i for i, h in enumerate(range(w.heads) if heads is None else heads)}
    for f, tok, h, ch in pos:
        if h in hmap:
            vals[f, tok, hmap[h], ch] *= OUTLIER_GAIN
    return (vals.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _sel_q(read, heads, fp4):
    """A read_ring / read_slot result of the low-precision formats restricted to `heads`."""
    if heads is None:
        return read
    codes, sc = read
    if fp4:
        return select_heads(codes, heads), (select_heads(sc[0], heads), sc[1][list(heads)])
    return select_heads(codes, heads), sc[list(heads)]


# the first and last of 40 states, each on its own pair of heads
HEADS_40_STATES = {0: (0, 39), 39: (13, 26)}


def test_tiny_fp8_two_states(torch):
    w = replace(PRESETS["tiny"], fp8=True, num_states=2, name="tiny_fp8")
    _run_fp8(torch, w, states=(0, 1))


def test_fp8_480x832_40_states(torch):
    _run_fp8(torch, PRESETS["fp8_480x832"], states=(0, 39), attend_blocks={1, 2, 5, 9, 17, 25}, rows=128,
             ring_frames=[0, 7], heads=HEADS_40_STATES)


# -- reference-image partition (attended first, exact, never evicted) ------------------

def test_tiny_reference_frames(torch):
    """Two reference frames (32 keys: one ragged tile) ahead of memory|window|current."""
    recs = _run(torch, PRESETS["tiny"], sink=2)
    assert sum(1 for r in recs if r[0] == "attend") == 15


def test_tiny_reference_frames_time_shift_invariance(torch):
    a, b = [], []
    _run(torch, PRESETS["tiny"], sink=2, t_offset=0, collect=a, max_blocks=8)
    _run(torch, PRESETS["tiny"], sink=2, t_offset=1000, collect=b, max_blocks=8)
    for (n, r, g0, ref), (_, _, g1, _) in zip(a, b):
        e = attention_errors(g1, g0)
        assert e["max"] <= 1e-2 and e["rel_l2"] <= 1e-2, (n, e)


def test_512_reference_frame(torch):
    _run(torch, PRESETS["512x512"], attend_blocks={1, 4, 13, 26}, rows=128, ring_frames=[0], sink=1, heads=HEADS8)


def test_720_reference_frame_ragged(torch):
    """1170-token frames: the reference segment ends in a ragged tile, as do the others."""
    _run(torch, PRESETS["720x416"], attend_blocks={1, 13, 38}, rows=128, ring_frames=[0], sink=1, heads=HEADS8)


def test_tiny_fp8_reference_frames_two_states(torch):
    """fp8 window/memory with bf16 reference frames, one per state."""
    w = replace(PRESETS["tiny"], fp8=True, num_states=2, name="tiny_fp8")
    _run_fp8(torch, w, states=(0, 1), sink=1)


# -- NVFP4 window and memory -------------------------------------------------

def test_tiny_nvfp4_two_states(torch):
    w = replace(PRESETS["tiny"], fp4=True, num_states=2, name="tiny_nvfp4")
    _run_fp8(torch, w, states=(0, 1))


def test_nvfp4_480x832_40_states(torch):
    _run_fp8(torch, PRESETS["nvfp4_480x832"], states=(0, 39), attend_blocks={1, 2, 5, 9, 17, 25}, rows=128,
             ring_frames=[0, 7], heads=HEADS_40_STATES)


# -- heavy tails: a few x16 values per frame and head in K and V ------------------------
# (the amax / scale / saturation paths see values far beyond the unit-variance inputs)

def test_tiny_fp8_outliers(torch):
    w = replace(PRESETS["tiny"], fp8=True, num_states=2, name="tiny_fp8")
    _run_fp8(torch, w, states=(0, 1), outliers=True)


def test_tiny_nvfp4_outliers(torch):
    w = replace(PRESETS["tiny"], fp4=True, num_states=2, name="tiny_nvfp4")
    _run_fp8(torch, w, states=(0, 1), outliers=True)


def test_fp8_480x832_outliers(torch):
    w = replace(PRESETS["fp8_480x832"], num_states=2)
    _run_fp8(torch, w, states=(0, 1), rows=128, ring_frames=[0, 7], heads={0: (0, 39), 1: (20,)}, outliers=True,
             max_blocks=5)


def test_nvfp4_480x832_outliers(torch):
    w = replace(PRESETS["nvfp4_480x832"], num_states=2)
    _run_fp8(torch, w, states=(0, 1), rows=128, ring_frames=[0, 7], heads={0: (0, 39), 1: (20,)}, outliers=True,
             max_blocks=5)


# -- odd head counts: the streaming kernels' (head, chunk) columns split into 128-thread
# slabs end inside a warp (9 heads x 16 chunks = 144 columns: a second slab of 16) ----

ODD_HEADS = Workload("odd_heads", 9, 128, 3, 7, 2, 2, 4, 3, 24, seed=9)


def test_odd_heads_stream(torch):
    _run(torch, ODD_HEADS)


def test_odd_heads_fp8_two_states(torch):
    _run_fp8(torch, replace(ODD_HEADS, fp8=True, num_states=2, name="odd_heads_fp8"), states=(0, 1))


def test_odd_heads_nvfp4_two_states(torch):
    _run_fp8(torch, replace(ODD_HEADS, fp4=True, num_states=2, name="odd_heads_nvfp4"), states=(0, 1))

"""C-ABI library on the host (no GPU): exports, argument checks, bookkeeping.

The library's integer bookkeeping (dry-run handles allocate no device memory
and launch nothing) must agree bit for bit with the oracle's stream state and
with the closed form of the eviction rule, for every block of every workload.
"""
import ctypes
import math
import re
from dataclasses import replace

import numpy as np
import pytest

import compressed_kv_cache_convkv_b200 as ckv
from compressed_kv_cache_convkv_b200.configs import PRESETS
from oracle import convkv_oracle as O


def _header_functions():
    import os
    text = open(os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "convkv.h")).read()
    return sorted(set(re.findall(r"^[\w\s\*]*?\b(convkv_\w+)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_symbol():
    lib = ckv.library()
    names = _header_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(ckv._SIGNATURES), "binding is missing a declared function"


def test_strerror():
    lib = ckv.library()
    assert lib.convkv_strerror(0) == b"ok"
    assert lib.convkv_strerror(ckv.ERR_DEVICE_TIMEOUT) == b"device wait timed out"


def _dry(w, **kw):
    return ckv.ConvKV(w.config(dry_run=True, **kw))


def test_invalid_configs_rejected():
    base = PRESETS["tiny"].config(dry_run=True)
    bad = [
        (base.with_(window_frames=3), ckv.ERR_INVALID_ARG),
        (base.with_(mem_slots=0), ckv.ERR_INVALID_ARG),
        (base.with_(evict_frames=4), ckv.ERR_UNSUPPORTED),
        (base.with_(head_dim=96), ckv.ERR_UNSUPPORTED),
        (base.with_(rope=(20, 22, 22)), ckv.ERR_UNSUPPORTED),
        (base.with_(num_states=0), ckv.ERR_INVALID_ARG),
        (base.with_(rope_theta=0.0), ckv.ERR_INVALID_ARG),
        (base.with_(grid_h=4096, grid_w=4096), ckv.ERR_UNSUPPORTED),
        (base.with_(sink_frames=-1), ckv.ERR_INVALID_ARG),
        (base.with_(kv_format=3), ckv.ERR_INVALID_ARG),
        (base.with_(kv_format=ckv.KV_NVFP4, compress_mode=ckv.COMPRESS_MEAN), ckv.ERR_UNSUPPORTED),
        (base.with_(sp_ranks=9), ckv.ERR_INVALID_ARG),
        (base.with_(sp_ranks=2, sp_rank=2), ckv.ERR_INVALID_ARG),
        (base.with_(sink_frames=100000), ckv.ERR_UNSUPPORTED),   # RoPE time table too large
    ]
    for cfg, code in bad:
        with pytest.raises(ckv.ConvKVError) as e:
            ckv.ConvKV(cfg)
        assert e.value.code == code, cfg
    # a real (non dry-run) conv handle needs weights; rejected before any CUDA call
    lib = ckv.library()
    assert lib.convkv_create(None, None) == ckv.ERR_INVALID_ARG
    c = PRESETS["tiny"].config()._c(0, 0)
    out = ctypes.c_void_p()
    assert lib.convkv_create(ctypes.byref(c), ctypes.byref(out)) == ckv.ERR_INVALID_ARG and not out


def test_call_order_and_argument_checks():
    h = _dry(PRESETS["tiny"])
    lib = ckv.library()
    assert lib.convkv_attend(h._h, None, None) == ckv.ERR_BAD_ORDER
    assert lib.convkv_append_block(h._h, None, None, 0) == ckv.ERR_INVALID_ARG
    assert lib.convkv_append_block(h._h, None, None, 3) == ckv.ERR_INVALID_ARG  # > max block
    c0 = h.counters()
    assert lib.convkv_append_block(h._h, None, None, 3) == ckv.ERR_INVALID_ARG
    assert h.counters() == c0, "a rejected call must leave the state unchanged"
    h.dry_append(2)
    assert lib.convkv_attend(h._h, None, None) == ckv.OK
    assert lib.convkv_read_slot(h._h, 0, 0, 0, None, None) == ckv.ERR_INVALID_ARG
    assert lib.convkv_append_block_host(h._h, None, None, 2) == ckv.ERR_INVALID_ARG
    assert lib.convkv_step_host(h._h, None, None, None, None, 2) == ckv.ERR_INVALID_ARG
    buf = ctypes.create_string_buffer(16)
    p = ctypes.cast(buf, ctypes.c_void_p)
    c1 = h.counters()
    # the host-buffer forms need device staging: dry-run handles refuse them untouched
    assert lib.convkv_step_host(h._h, p, p, p, p, 2) == ckv.ERR_BAD_ORDER
    assert lib.convkv_step_host(h._h, p, p, p, p, 3) == ckv.ERR_INVALID_ARG   # > max block
    assert lib.convkv_append_block_host(h._h, p, p, 2) == ckv.ERR_BAD_ORDER
    assert lib.convkv_step_host_async(h._h, p, p, p, p, 2) == ckv.ERR_BAD_ORDER
    assert lib.convkv_step_host_async(h._h, None, p, p, p, 2) == ckv.ERR_INVALID_ARG
    assert lib.convkv_step_host_async(h._h, p, p, p, p, 0) == ckv.ERR_INVALID_ARG
    assert lib.convkv_sync(h._h) == ckv.OK and lib.convkv_sync(None) == ckv.ERR_INVALID_ARG
    assert h.counters() == c1
    assert lib.convkv_state_bytes(h._h) == 0 and h.launch_count() == 0
    lib.convkv_destroy(None)


def _oracle_layout(st):
    return [(int(p), int(s), int(t)) for p, s, t in st.layout()]


@pytest.mark.parametrize("name", ["tiny", "512x512", "720x416", "fp8_480x832", "nvfp4_480x832"])
def test_bookkeeping_matches_oracle_every_block(name):
    w = PRESETS[name]
    h = _dry(w)
    cfg = O.OracleConfig(H=1, D=6, grid_h=1, grid_w=1, window=w.window_frames, mem_slots=w.mem_slots)
    st = O.OracleStream(cfg, np.zeros((2, 1, 6, 6, 5)))
    R = w.window_frames + max(w.first_block_frames, w.block_frames)
    for n, b in enumerate(w.block_sizes()):
        h.dry_append(b)
        ev = st.append(np.zeros((b, 1, 1, 6)), np.zeros((b, 1, 1, 6)))
        c = h.counters()
        assert (c["P"], c["E"], c["S"], c["m"], c["w"], c["b"], c["blocks"], c["groups"]) == \
            (st.P, st.E, st.S, st.m, st.w_frames, b, n + 1, len(ev))
        lay = h.layout()
        assert [tuple(r) for r in lay[:, [0, 1, 3]]] == _oracle_layout(st)
        # physical slots: memory position = slot mod C, ring slot = frame mod R
        for part, src, phys, _ in lay:
            if part == 2 and (w.fp8 or w.fp4):   # low precision: the current block sits in bf16 staging
                assert phys == src - st.P
            else:
                assert phys == (src % w.mem_slots if part == 0 else src % R)


@pytest.mark.parametrize("name,sink", [("tiny", 2), ("512x512", 1), ("fp8_480x832", 1)])
def test_reference_frames_lead_the_layout(name, sink):
    """Reference-image frames come first at time 0..r-1, never move, and shift every other
    time index by r; the rest of the layout is the sink-free one."""
    w = PRESETS[name]
    h = _dry(w, sink_frames=sink)
    lib = ckv.library()
    cfg = O.OracleConfig(H=1, D=6, grid_h=1, grid_w=1, window=w.window_frames, mem_slots=w.mem_slots)
    st = O.OracleStream(cfg, np.zeros((2, 1, 6, 6, 5)))
    st.set_sink(np.zeros((sink, 1, 1, 6)), np.zeros((sink, 1, 1, 6)))
    h.dry_append(w.block_sizes()[0])
    assert lib.convkv_attend(h._h, None, None) == ckv.ERR_BAD_ORDER      # reference not given yet
    h.set_sink(None, None)
    assert lib.convkv_attend(h._h, None, None) == ckv.OK
    st.append(np.zeros((w.block_sizes()[0], 1, 1, 6)), np.zeros((w.block_sizes()[0], 1, 1, 6)))
    for b in w.block_sizes()[1:]:
        h.dry_append(b)
        st.append(np.zeros((b, 1, 1, 6)), np.zeros((b, 1, 1, 6)))
        lay = h.layout()
        assert [tuple(r) for r in lay[:, [0, 1, 3]]] == _oracle_layout(st)
        assert [tuple(r) for r in lay[:sink]] == [(3, i, i, i) for i in range(sink)]
        assert list(lay[:, 3]) == list(range(len(lay)))


def test_set_sink_needs_reference_frames():
    h = _dry(PRESETS["tiny"])
    assert ckv.library().convkv_set_sink(h._h, None, None) == ckv.ERR_BAD_ORDER
    assert ckv.library().convkv_set_sink(None, None, None) == ckv.ERR_INVALID_ARG


def test_soak_bookkeeping_closed_form_and_constant_footprint():
    w = PRESETS["soak"]
    h = _dry(w)
    W, C = w.window_frames, w.mem_slots
    total = 0
    sizes = w.block_sizes()
    assert len(sizes) == 2251 and sum(sizes) == 18000
    max_keys = 0
    for b in sizes:
        h.dry_append(b)
        c = h.counters()
        E = 5 * math.ceil(max(0, total - W) / 5)
        S = E // 5
        assert (c["P"], c["E"], c["S"], c["m"], c["w"]) == (total, E, S, min(S, C), total - E)
        lay = h.layout()
        assert list(lay[:, 3]) == list(range(len(lay)))          # reset time indices 0..n-1
        assert list(lay[lay[:, 0] == 0, 1]) == list(range(S - min(S, C), S))
        total += b
        max_keys = max(max_keys, len(lay))
    assert max_keys <= C + W + max(w.first_block_frames, w.block_frames)


def test_first_conv_at_block_3_for_512():
    h = _dry(PRESETS["512x512"])
    groups = []
    for b in PRESETS["512x512"].block_sizes()[:4]:
        h.dry_append(b)
        groups.append(h.counters()["groups"])
    assert groups[:3] == [0, 0, 1]


def test_sequence_parallel_argument_checks():
    """Host-side checks of the sequence-parallel forms (no CUDA call is reached)."""
    lib = ckv.library()
    w = PRESETS["tiny"]
    plain = _dry(w)
    two = (ctypes.c_void_p * 2)(1, 2)
    # the SP forms need a handle created with sp_ranks >= 2
    assert lib.convkv_append_block_sp(plain._h, two, two, 2) == ckv.ERR_INVALID_ARG
    assert lib.convkv_attend_sp(plain._h, two, two) == ckv.ERR_INVALID_ARG
    sp = _dry(w, heads=1, sp_ranks=2, sp_rank=1)
    assert lib.convkv_attend_sp(sp._h, two, two) == ckv.ERR_BAD_ORDER      # nothing appended yet
    assert lib.convkv_append_block_sp(sp._h, two, two, 0) == ckv.ERR_INVALID_ARG
    assert lib.convkv_append_block_sp(sp._h, two, two, 2) == ckv.OK        # dry run: bookkeeping only
    assert lib.convkv_attend_sp(sp._h, two, two) == ckv.OK
    assert sp.counters()["b"] == 2
    # the IPC helpers reject null arguments before touching CUDA
    assert lib.convkv_ipc_export(None, None, None) == ckv.ERR_INVALID_ARG
    assert lib.convkv_ipc_open(None, None) == ckv.ERR_INVALID_ARG
    assert lib.convkv_ipc_close(None) == ckv.ERR_INVALID_ARG


def test_low_precision_formats_share_the_bookkeeping():
    """e4m3 and NVFP4 handles keep the bf16 bookkeeping; only the current block's
    physical slots (staging) differ."""
    w = PRESETS["fp8_480x832"]
    hs = {fmt: _dry(w, kv_format=fmt) for fmt in (ckv.KV_BF16, ckv.KV_FP8_E4M3, ckv.KV_NVFP4)}
    for b in w.block_sizes()[:12]:
        for h in hs.values():
            h.dry_append(b)
        lays = {fmt: h.layout() for fmt, h in hs.items()}
        ref = lays[ckv.KV_BF16]
        for fmt in (ckv.KV_FP8_E4M3, ckv.KV_NVFP4):
            assert np.array_equal(lays[fmt][:, [0, 1, 3]], ref[:, [0, 1, 3]])
            cur = lays[fmt][:, 0] == 2
            assert list(lays[fmt][cur, 2]) == list(range(int(cur.sum())))


@pytest.mark.parametrize("step", [0, 1, 2])
def test_failed_append_leaves_the_state_unchanged(step):
    """A launch failure injected on the host at one step of an append (conv, time-table
    upload, ring append) leaves counters and layout as they were; attends are refused
    until an append succeeds, and the stream then continues exactly like a stream that
    never failed."""
    w = PRESETS["512x512"]
    h, ref = _dry(w), _dry(w)
    lib = ckv.library()
    sizes = w.block_sizes()
    # blocks 1..2 need no conv; block 3 runs the first one (step 0 is then the conv)
    n_before = 2 if step == 0 else 4
    for b in sizes[:n_before]:
        h.dry_append(b)
        ref.dry_append(b)
    before = (h.counters(), h.layout().tolist())
    assert lib.convkv_debug_fail_step(h._h, step) == ckv.OK
    rc = lib.convkv_append_block(h._h, None, None, sizes[n_before])
    assert rc == ckv.ERR_CUDA
    assert lib.convkv_last_cuda_error(h._h) != 0
    assert (h.counters(), h.layout().tolist()) == before
    assert lib.convkv_attend(h._h, None, None) == ckv.ERR_BAD_ORDER
    for b in sizes[n_before:n_before + 6]:
        h.dry_append(b)
        ref.dry_append(b)
        assert h.counters() == ref.counters()
        assert h.layout().tolist() == ref.layout().tolist()
    assert lib.convkv_attend(h._h, None, None) == ckv.OK
    assert lib.convkv_debug_fail_step(h._h, -2) == ckv.ERR_INVALID_ARG


def test_noalloc_quantiser_rejects_misaligned_pointers_before_any_work():
    """x is read in 16-byte vectors, codes written in 8-byte vectors, scales as fp32:
    a misaligned pointer returns INVALID_ARG before any CUDA call (the addresses
    here are never dereferenced)."""
    lib = ckv.library()
    good = 1 << 20
    for x, c, s in [(good + 8, good, good), (good, good + 4, good), (good, good, good + 2)]:
        assert lib.convkv_quantize_e4m3_noalloc(x, c, s, 1, 16, 2, 64, None) == ckv.ERR_INVALID_ARG


def _plan(w, queued=False, **kw):
    return _dry(w, host_io=True, **kw).host_chunks(queued).tolist()


def test_host_chunk_plan_covers_every_state_and_head_once():
    """The host-buffer chunk plan (convkv_host_chunks, computed on the host for 148
    SMs): every (state, head) pair lies in exactly one chunk, in stream order; whole
    states with several states, ranges of heads with one state."""
    cases = [(PRESETS[n], {}) for n in ("tiny", "512x512", "720x416", "fp8_480x832", "nvfp4_480x832")]
    cases += [(replace(PRESETS["fp8_480x832"], num_states=s), {}) for s in (1, 2, 7, 8, 13)]
    cases += [(replace(PRESETS["tiny"], num_states=s), {}) for s in (1, 2, 3, 5)]
    cases += [(replace(PRESETS["512x512"], num_states=s), {}) for s in (2, 40)]
    for (w, kw), queued in [(c, q) for c in cases for q in (False, True)]:
        plan = _plan(w, queued, **kw)
        H, S = w.heads, w.num_states
        seen = np.zeros((S, H), dtype=int)
        for g0, n, h0, nh in plan:
            assert n >= 1 and nh >= 1
            if nh < H:
                assert n == 1, (w.name, plan)
            seen[g0:g0 + n, h0:h0 + nh] += 1
        assert (seen == 1).all(), (w.name, S, plan)
        flat = [(g0, h0) for g0, _, h0, _ in plan]
        assert flat == sorted(flat), plan
        if S > 1:
            assert all(nh == H for _, _, _, nh in plan)
            sizes = [n for _, n, _, _ in plan]
            if not queued:
                assert sizes[0] == 1 and sizes[-1] == 1, sizes
            else:
                assert len(sizes) >= 2 and len(set(sizes[:-1])) <= 1 and sizes[-1] <= sizes[0], sizes
        elif H > 1:
            assert len(plan) >= 2
    # a handle without host buffers has no plan
    assert _dry(PRESETS["tiny"]).host_chunks().shape == (0, 4)


def test_host_chunk_plan_fills_waves_at_the_bench_shapes():
    """At the bench shapes the plan's attention grids fill their waves of 148 SMs:
    480x832 x 40 states in steady chunks of 4 states (4 x 1,960 CTAs = 53 waves, 0.06 %
    idle); one state in ranges of heads that make one wave each: 4 heads x 32 CTAs at
    512x512 (86 % full), 4 x 37 at 720x416 (full), 3 x 49 at 480x832 (99 %).  Head
    ranges are at least 512 bytes per token row."""
    fp8 = _plan(PRESETS["fp8_480x832"])
    assert [n for _, n, _, _ in fp8] == [1, 1, 1, 2, 2, 3, 4, 4, 4, 4, 4, 4, 3, 2, 1]
    assert [n for _, n, _, _ in _plan(PRESETS["fp8_480x832"], True)] == [7] * 5 + [5]
    assert _plan(PRESETS["512x512"], True) == _plan(PRESETS["512x512"])
    assert max(n for _, n, _, _ in fp8) <= 7        # the e4m3 dequantisation group
    assert _plan(PRESETS["512x512"]) == [[0, 1, h, 4] for h in range(0, 40, 4)]
    assert _plan(PRESETS["720x416"]) == [[0, 1, h, 4] for h in range(0, 40, 4)]
    one = _plan(replace(PRESETS["fp8_480x832"], num_states=1))
    assert one == [[0, 1, h, 3] for h in range(0, 39, 3)] + [[0, 1, 39, 1]]
    for w in (PRESETS["512x512"], PRESETS["720x416"], replace(PRESETS["fp8_480x832"], num_states=1)):
        per_head = -(-w.block_frames * w.T // 256)
        nh = _plan(w)[0][3]
        ctas = per_head * nh
        assert ctas <= 148 and ctas / 148 >= 0.85
        assert nh * w.head_dim * 2 >= 512

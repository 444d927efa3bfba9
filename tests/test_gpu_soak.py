"""Hour-scale soak: the 512x512 shape streamed for 18,000 latent frames (2,251 blocks).

Checks, on one B200:
  * constant footprint: convkv_state_bytes and the device's free bytes are the same
    after every block (SoulX-LiveAct blog, "Streaming Pipeline": the KV cache size is
    the same for one minute or one hour);
  * indices bit-exact at every block against the closed form of the eviction rule;
  * outputs and compressed slots against a running oracle for the first 500 frames;
  * outputs at 20 blocks drawn with seed 3 from blocks 64..2251, where the oracle
    rebuilds that block's state from the closed form and regenerates only the frames
    it needs (memory slot k is the conv of frames [5k, 5k+5)).
"""
import math

import numpy as np
import pytest

import seeded_inputs as si
from compressed_kv_cache_convkv_b200.configs import PRESETS
from oracle import convkv_oracle as O
from streams import (bf16_tensor_to_f64, check_attention, check_slot, device_frames, device_weights,
                     host_frames, oracle_for, sample_rows, select_heads)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

# Heads the oracle evaluates (heads are independent through the whole step, so a head
# subset of the oracle gives exactly those heads' values): first, last and two between.
HEADS = (0, 13, 26, 39)


@pytest.fixture(scope="module")
def torch():
    import torch as t
    assert t.cuda.is_available(), "GPU tests need a CUDA device"
    from compressed_kv_cache_convkv_b200 import build
    build.build()
    si.build(device=True)
    return t


def _closed_form(P, W, C):
    E = 5 * math.ceil(max(0, P - W) / 5)
    S = E // 5
    return E, P - E, S, min(S, C)


def _replayed_oracle(w, P, b, F):
    """Oracle state of the block that starts at stream frame F (= P promoted frames),
    rebuilt from the closed form with only the frames it needs."""
    E, wn, S, m = _closed_form(P, w.window_frames, w.mem_slots)
    st = oracle_for(w, heads=HEADS)
    fr = lambda t, f0, n: si.bf16_bits_to_f64(host_frames(w, t, 0, f0, n, HEADS))
    for k in range(S - m, S):
        kk, vv = fr(si.K, 5 * k, 5), fr(si.V, 5 * k, 5)
        st.memory.append(O._Frame(O.round_to_bf16(O.conv_compress(kk, st.w[0])),
                                  O.round_to_bf16(O.conv_compress(vv, st.w[1])), k))
    kw, vw = fr(si.K, E, wn), fr(si.V, E, wn)
    st.window = [O._Frame(kw[i], vw[i], E + i) for i in range(wn)]
    kc, vc = fr(si.K, F, b), fr(si.V, F, b)
    st.current = [O._Frame(kc[i], vc[i], F + i) for i in range(b)]
    st.P, st.E, st.S = P, E, S
    return st


def _rows(out, r):
    """Selected output rows of the oracle's heads, gathered on the host (no device
    allocation inside the loop)."""
    return select_heads(bf16_tensor_to_f64(out[0].cpu()[r]), HEADS)


def test_soak_18000_frames(torch):
    import compressed_kv_cache_convkv_b200 as ckv
    w = PRESETS["soak"]
    sizes = w.block_sizes()
    assert len(sizes) == 2251 and sum(sizes) == 18000
    cfg = w.config()
    h = ckv.ConvKV(cfg, device_weights(w, torch))
    bmax = cfg.max_block
    # inputs are regenerated on the device into these buffers every block (no allocation in the loop)
    bufs = {t: torch.empty((1, bmax * w.T, w.heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
            for t in (si.Q, si.K, si.V)}
    out_buf = torch.empty_like(bufs[si.Q])
    rng = np.random.default_rng(w.seed)
    samples = set(int(x) for x in rng.choice(np.arange(64, len(sizes) + 1), size=20, replace=False))
    running = oracle_for(w, heads=HEADS)
    state_bytes = h.state_bytes()
    free0 = None
    F = 0
    checked = 0
    for n, b in enumerate(sizes, start=1):
        view = {t: bufs[t][:, : b * w.T] for t in bufs}
        for t in (si.Q, si.K, si.V):
            device_frames(w, t, F, b, torch, out=view[t])
        h.append(view[si.K], view[si.V])
        out = out_buf[:, : b * w.T]
        h.attend(view[si.Q], out)
        # footprint
        assert h.state_bytes() == state_bytes
        torch.cuda.synchronize()
        free = torch.cuda.mem_get_info()[0]
        if free0 is None:
            free0 = free
        assert free == free0, f"free device memory changed at block {n}"
        # indices: closed form, bit-exact
        E, wn, S, m = _closed_form(F, w.window_frames, w.mem_slots)
        c = h.counters()
        assert (c["P"], c["E"], c["S"], c["m"], c["w"], c["b"]) == (F, E, S, m, wn, b), n
        lay = h.layout()
        assert list(lay[:, 0]) == [0] * m + [1] * wn + [2] * b
        assert list(lay[:, 1]) == list(range(S - m, S)) + list(range(E, F)) + list(range(F, F + b))
        assert list(lay[:, 3]) == list(range(m + wn + b))
        # running oracle over the first 500 frames
        if F < 500:
            kh, vh = (si.bf16_bits_to_f64(host_frames(w, t, 0, F, b, HEADS)) for t in (si.K, si.V))
            ev = running.append(kh, vh)
            for e in ev[-cfg.mem_slots:]:
                gk, _ = h.read_slot(0, 0, e.slot % cfg.mem_slots)
                check_slot(si.bf16_bits_to_f64(select_heads(gk, HEADS)),
                           running.memory_slot(running.m - (running.S - e.slot))[0], f"soak K slot {e.slot}")
            if n % 4 == 1 or n == 63:
                qh = si.bf16_bits_to_f64(host_frames(w, si.Q, 0, F, b, HEADS))
                r = sample_rows(w, b, 64, rng)
                ref, _ = running.attend(qh, rows=r)
                check_attention(_rows(out, r), ref, what=f"soak block {n}")
                checked += 1
        elif F >= 500 and running is not None:
            running = None        # release the running state
        # replayed oracle at sampled late blocks
        if n in samples:
            st = _replayed_oracle(w, F, b, F)
            assert [tuple(x) for x in st.layout()] == [tuple(x) for x in lay[:, [0, 1, 3]]]
            qh = si.bf16_bits_to_f64(host_frames(w, si.Q, 0, F, b, HEADS))
            r = sample_rows(w, b, 64, rng)
            ref, _ = st.attend(qh, rows=r)
            check_attention(_rows(out, r), ref, what=f"soak replayed block {n}")
            checked += 1
        F += b
    assert h.status() == 0
    assert checked >= 16 + 20
    h.close()

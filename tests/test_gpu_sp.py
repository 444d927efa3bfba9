"""Sequence-parallel form on one GPU: G ranks emulated by G handles.

Each handle owns H/G heads and reads its rows from the G sequence shards (here all
local buffers; on a multi-GPU node they are peer memory).  The fused gather (append,
queries) and scatter (outputs) must reproduce the plain all-heads path bit for bit:
every head runs the same arithmetic, only the addressing differs.  The plain path
is itself checked against the fp64 oracle (test_gpu_parity.py); a few blocks are
checked against the oracle here as well.
"""
from dataclasses import replace

import numpy as np
import pytest

import seeded_inputs as si
from compressed_kv_cache_convkv_b200.configs import PRESETS
from compressed_kv_cache_convkv_b200.sp import head_range, shard_rows, split_block
from streams import (bf16_tensor_to_f64, check_attention, device_frames, device_weights, host_frames, oracle_for,
                     select_heads)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    assert t.cuda.is_available(), "GPU tests need a CUDA device"
    from compressed_kv_cache_convkv_b200 import build
    build.build()
    si.build(device=True)
    return t


def _run_sp(torch, w, G, max_blocks=None, oracle_blocks=(), sink=0, rows=64, heads=None):
    import compressed_kv_cache_convkv_b200 as ckv
    H, T = w.heads, w.T
    weights = device_weights(w, torch)
    cfg = w.config(sink_frames=sink)
    plain = ckv.ConvKV(cfg, weights)
    ranks = []
    for g in range(G):
        hr = head_range(H, G, g)
        ranks.append((hr, ckv.ConvKV(cfg.with_(heads=len(hr), sp_ranks=G, sp_rank=g),
                                     weights[:, :, hr.start:hr.stop].contiguous())))
    st = oracle_for(w, heads=heads) if oracle_blocks else None
    if sink:
        rk, rv = device_frames(w, si.RK, 0, sink, torch), device_frames(w, si.RV, 0, sink, torch)
        plain.set_sink(rk, rv)
        for hr, hd in ranks:
            hd.set_sink(rk[:, :, hr.start:hr.stop].contiguous(), rv[:, :, hr.start:hr.stop].contiguous())
        if st is not None:
            st.set_sink(si.bf16_bits_to_f64(host_frames(w, si.RK, 0, 0, sink, heads)),
                        si.bf16_bits_to_f64(host_frames(w, si.RV, 0, 0, sink, heads)))
    rng = np.random.default_rng(w.seed)
    R = cfg.ring_frames
    F = 0
    for n, b in enumerate(w.block_sizes()[: max_blocks or None], start=1):
        kd, vd, qd = (device_frames(w, t, F, b, torch) for t in (si.K, si.V, si.Q))
        plain.append(kd, vd)
        ref = plain.attend(qd)
        ks, vs, qs = ([x.contiguous() for x in split_block(t, G)] for t in (kd, vd, qd))
        assert [x.shape[1] for x in qs] == list(np.diff(shard_rows(b * T, G)))
        outs = [torch.full_like(x, float("nan")) for x in qs]
        for _, hd in ranks:
            hd.append_sp(ks, vs, b)
        for _, hd in ranks:
            hd.attend_sp(qs, outs)
        out = torch.cat(outs, dim=1)
        assert torch.equal(out, ref), f"{w.name} G={G} block {n}: sequence-parallel output differs from the plain path"
        # the gathered ring frames are the plain ring's head slices, bit for bit
        for f in (0, b - 1):
            pk, _ = plain.read_ring(0, 0, (F + f) % R)
            pv, _ = plain.read_ring(0, 1, (F + f) % R)
            for hr, hd in ranks:
                gk, _ = hd.read_ring(0, 0, (F + f) % R)
                gv, _ = hd.read_ring(0, 1, (F + f) % R)
                assert np.array_equal(gk, pk.reshape(T, H, -1)[:, hr.start:hr.stop].reshape(gk.shape)), n
                assert np.array_equal(gv, pv.reshape(T, H, -1)[:, hr.start:hr.stop].reshape(gv.shape)), n
        if st is not None:
            kh, vh, qh = (host_frames(w, t, 0, F, b, heads) for t in (si.K, si.V, si.Q))
            st.append(si.bf16_bits_to_f64(kh), si.bf16_bits_to_f64(vh))
            if n in oracle_blocks:
                r = np.sort(rng.choice(b * T, size=min(rows, b * T), replace=False))
                o, _ = st.attend(si.bf16_bits_to_f64(qh), rows=r)
                check_attention(select_heads(bf16_tensor_to_f64(out[0][torch.as_tensor(r, device="cuda")]), heads),
                                o, what=f"{w.name} G={G} block {n}")
        F += b
    assert plain.status() == 0 and all(hd.status() == 0 for _, hd in ranks)
    plain.close()
    for _, hd in ranks:
        hd.close()


def test_sp_tiny_two_ranks(torch):
    _run_sp(torch, PRESETS["tiny"], 2, oracle_blocks={1, 5, 9, 15}, rows=32)


def test_sp_512_four_ranks(torch):
    _run_sp(torch, PRESETS["512x512"], 4, max_blocks=6, oracle_blocks={6}, heads=(0, 9, 10, 19, 20, 29, 30, 39))


def test_sp_720_eight_ranks_uneven_rows_with_reference(torch):
    """1170-token frames: shard boundaries fall inside frames and tiles (7020 rows / 8)."""
    _run_sp(torch, PRESETS["720x416"], 8, max_blocks=5, sink=1)


def test_sp_tiny_fp8_two_states(torch):
    w = replace(PRESETS["tiny"], fp8=True, num_states=2, name="tiny_fp8")
    _run_sp(torch, w, 2, max_blocks=10)

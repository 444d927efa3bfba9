"""The host-buffer entry points (convkv_append_block_host / convkv_attend_host /
convkv_step_host / convkv_step_host_async) against the device-buffer ones, on the GPU.

The host forms copy their inputs in by chunks on a copy stream, start each chunk's
kernels as soon as its copy lands, and copy each chunk's outputs back while later
chunks compute; convkv_step_host does an append and an attend in one such pipelined
call.  The kernels and their arithmetic are the same as in the device forms, so the
outputs must be identical bit for bit, for several chunks: a bf16 handle of 3 states
(three chunks), an e4m3 handle of 8 states at 480x832 (chunks of 1 to 2 states, under
the 4 GiB dequantisation scratch), and handles of one state, whose chunks are ranges
of heads copied with strided copies (bf16, e4m3 and NVFP4; ranges of 4 heads at
512x512, of 3 heads and a last one of 1 at 480x832, of one head in the tiny shape).
"""
from dataclasses import replace

import numpy as np
import pytest

import seeded_inputs as si
from compressed_kv_cache_convkv_b200.configs import PRESETS
from streams import device_frames, device_weights

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    assert t.cuda.is_available(), "GPU tests need a CUDA device"
    from compressed_kv_cache_convkv_b200 import build
    build.build()
    si.build(device=True)
    return t


def _block(torch, w, tid, frame0, frames):
    x = torch.empty((w.num_states, frames * w.T, w.heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    fe = w.T * w.heads * w.head_dim
    stream = torch.cuda.current_stream().cuda_stream
    for s in range(w.num_states):
        si.frames_device(x[s].data_ptr(), w.seed, tid, s, frame0, frames, fe, 1.0, stream)
    return x


def _pinned(torch, x):
    h = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    h.copy_(x)
    return h


@pytest.mark.parametrize("name,states,blocks,kw", [
    ("tiny", 3, 12, {}),
    ("fp8_480x832", 8, 5, {}),
    # one state: chunks of heads (strided copies), in every storage format
    ("tiny", 1, 12, {}),
    ("tiny", 1, 8, {"fp8": True}),
    ("tiny", 1, 8, {"fp4": True}),
    ("512x512", 1, 5, {}),
    ("fp8_480x832", 1, 4, {}),
    ("nvfp4_480x832", 1, 4, {}),
])
def test_host_buffers_match_device_buffers(torch, name, states, blocks, kw):
    import compressed_kv_cache_convkv_b200 as ckv
    w = replace(PRESETS[name], num_states=states, **kw)
    weights = device_weights(w, torch)
    dev = ckv.ConvKV(w.config(), weights)
    hio = ckv.ConvKV(w.config(host_io=True), weights)
    fused = ckv.ConvKV(w.config(host_io=True), weights)
    frame0 = 0
    for i, frames in enumerate(w.block_sizes()[:blocks]):
        q, k, v = (_block(torch, w, tid, frame0, frames) for tid in (si.Q, si.K, si.V))
        frame0 += frames
        dev.append(k, v)
        o_dev = dev.attend(q)
        qh, kh, vh = (_pinned(torch, x) for x in (q, k, v))
        oh = torch.empty(qh.shape, dtype=qh.dtype, pin_memory=True)
        of = torch.empty(qh.shape, dtype=qh.dtype, pin_memory=True)
        hio.append_host(kh, vh)
        hio.attend_host(qh, oh)
        fused.step_host(kh, vh, qh, of)
        torch.cuda.synchronize()
        a = o_dev.view(torch.int16).cpu().numpy()
        assert np.array_equal(a, oh.view(torch.int16).numpy()), (name, i, "append_host + attend_host")
        assert np.array_equal(a, of.view(torch.int16).numpy()), (name, i, "step_host")
        assert dev.counters() == hio.counters() == fused.counters()
    assert dev.status() == 0 and hio.status() == 0 and fused.status() == 0
    for h in (dev, hio, fused):
        h.close()


@pytest.mark.parametrize("step", [0, 1, 2])
def test_step_host_failure_rolls_back_and_recovers(torch, step):
    """A launch failure injected on the host at one step of convkv_step_host's append
    (conv, time-table upload, ring append) leaves the counters as before the call and
    refuses attends; repeating the same step then gives the device path's outputs bit
    for bit (the failed call's partial work is rewritten)."""
    import compressed_kv_cache_convkv_b200 as ckv
    w = replace(PRESETS["tiny"], fp8=True, num_states=3, name="tiny_fp8")
    weights = device_weights(w, torch)
    dev = ckv.ConvKV(w.config(), weights)
    hio = ckv.ConvKV(w.config(host_io=True), weights)
    lib = ckv.library()
    frame0 = 0
    for i, frames in enumerate(w.block_sizes()[:8]):
        q, k, v = (_block(torch, w, tid, frame0, frames) for tid in (si.Q, si.K, si.V))
        frame0 += frames
        dev.append(k, v)
        o_dev = dev.attend(q)
        qh, kh, vh = (_pinned(torch, x) for x in (q, k, v))
        oh = torch.empty(qh.shape, dtype=qh.dtype, pin_memory=True)
        if i == 5:
            # block 5 evicts a group, so all three append steps run
            before = hio.counters()
            assert lib.convkv_debug_fail_step(hio._h, step) == ckv.OK
            rc = lib.convkv_step_host(hio._h, kh.data_ptr(), vh.data_ptr(), qh.data_ptr(), oh.data_ptr(), frames)
            assert rc == ckv.ERR_CUDA
            assert hio.counters() == before
            assert lib.convkv_attend_host(hio._h, qh.data_ptr(), oh.data_ptr()) == ckv.ERR_BAD_ORDER
        hio.step_host(kh, vh, qh, oh)
        torch.cuda.synchronize()
        assert np.array_equal(o_dev.view(torch.int16).cpu().numpy(), oh.view(torch.int16).numpy()), (step, i)
        assert dev.counters() == hio.counters()
    assert dev.status() == 0 and hio.status() == 0
    dev.close()
    hio.close()


@pytest.mark.parametrize("name,states,blocks,kw", [
    ("tiny", 3, 10, {}),
    ("tiny", 1, 8, {"fp8": True}),
    ("512x512", 1, 5, {}),
    ("fp8_480x832", 4, 3, {}),
])
def test_queued_steps_match_device_buffers(torch, name, states, blocks, kw):
    """Host-buffer steps queued back to back (convkv_step_host_async, one convkv_sync at
    the end): each chunk's copy in waits only for the previous step's kernels and copy
    back of that chunk, so steps overlap.  Every step's outputs must equal the device
    path's bit for bit.  At 512x512 the first block has 6 frames and the others 8,
    which moves every chunk's staging region: there the second step's copies must wait
    for the whole first step."""
    import compressed_kv_cache_convkv_b200 as ckv
    w = replace(PRESETS[name], num_states=states, **kw)
    weights = device_weights(w, torch)
    dev = ckv.ConvKV(w.config(), weights)
    hio = ckv.ConvKV(w.config(host_io=True), weights)
    frame0 = 0
    expected, queued = [], []
    for frames in w.block_sizes()[:blocks]:
        q, k, v = (_block(torch, w, tid, frame0, frames) for tid in (si.Q, si.K, si.V))
        frame0 += frames
        dev.append(k, v)
        expected.append(dev.attend(q))
        qh, kh, vh = (_pinned(torch, x) for x in (q, k, v))
        oh = torch.empty(qh.shape, dtype=qh.dtype, pin_memory=True)
        hio.step_host_async(kh, vh, qh, oh)
        queued.append((qh, kh, vh, oh))   # every queued step's buffers stay alive
    hio.sync()
    torch.cuda.synchronize()
    for i, (o_dev, (_, _, _, oh)) in enumerate(zip(expected, queued)):
        assert np.array_equal(o_dev.view(torch.int16).cpu().numpy(), oh.view(torch.int16).numpy()), (name, i)
    assert dev.counters() == hio.counters()
    assert dev.status() == 0 and hio.status() == 0
    dev.close()
    hio.close()


@pytest.mark.parametrize("name,states", [("512x512", 1), ("tiny", 3)])
def test_host_buffers_with_reference_frames(torch, name, states):
    """With a reference-image partition (one frame, attended first and never evicted)
    the host forms still equal the device form bit for bit: the reference keys enter
    every chunk's attention through their own tensor maps, with head ranges (one
    state) and whole-state chunks (three states), synchronous and queued."""
    import compressed_kv_cache_convkv_b200 as ckv
    w = replace(PRESETS[name], num_states=states)
    weights = device_weights(w, torch)
    hs = [ckv.ConvKV(w.config(sink_frames=1, **kw), weights) for kw in ({}, {"host_io": True}, {"host_io": True})]
    rk, rv = device_frames(w, si.RK, 0, 1, torch), device_frames(w, si.RV, 0, 1, torch)
    for h in hs:
        h.set_sink(rk, rv)
    dev, sync, queued = hs
    frame0 = 0
    expected, outs = [], []
    for frames in w.block_sizes()[:5]:
        q, k, v = (_block(torch, w, tid, frame0, frames) for tid in (si.Q, si.K, si.V))
        frame0 += frames
        dev.append(k, v)
        expected.append(dev.attend(q))
        qh, kh, vh = (_pinned(torch, x) for x in (q, k, v))
        o1 = torch.empty(qh.shape, dtype=qh.dtype, pin_memory=True)
        o2 = torch.empty(qh.shape, dtype=qh.dtype, pin_memory=True)
        sync.step_host(kh, vh, qh, o1)
        queued.step_host_async(kh, vh, qh, o2)
        outs.append((qh, kh, vh, o1, o2))
    queued.sync()
    torch.cuda.synchronize()
    for i, (o_dev, (_, _, _, o1, o2)) in enumerate(zip(expected, outs)):
        a = o_dev.view(torch.int16).cpu().numpy()
        assert np.array_equal(a, o1.view(torch.int16).numpy()), (name, i, "step_host")
        assert np.array_equal(a, o2.view(torch.int16).numpy()), (name, i, "step_host_async")
    for h in hs:
        assert h.status() == 0
        h.close()


def test_queued_step_failure_rolls_back_and_recovers(torch):
    """A launch failure injected on the host while a queued step is being queued (behind
    two queued steps still in flight): the call waits everything out, restores the
    counters and refuses attends; the earlier queued steps' outputs are complete and
    correct, and queueing the same step again gives the device path's outputs."""
    import compressed_kv_cache_convkv_b200 as ckv
    w = replace(PRESETS["tiny"], fp8=True, num_states=3, name="tiny_fp8")
    weights = device_weights(w, torch)
    dev = ckv.ConvKV(w.config(), weights)
    hio = ckv.ConvKV(w.config(host_io=True), weights)
    lib = ckv.library()
    frame0 = 0
    expected, queued = [], []
    for i, frames in enumerate(w.block_sizes()[:8]):
        q, k, v = (_block(torch, w, tid, frame0, frames) for tid in (si.Q, si.K, si.V))
        frame0 += frames
        dev.append(k, v)
        expected.append(dev.attend(q))
        qh, kh, vh = (_pinned(torch, x) for x in (q, k, v))
        oh = torch.empty(qh.shape, dtype=qh.dtype, pin_memory=True)
        if i == 5:
            # block 5 evicts a group, so the conv runs: fail it
            before = hio.counters()
            assert lib.convkv_debug_fail_step(hio._h, 0) == ckv.OK
            rc = lib.convkv_step_host_async(hio._h, kh.data_ptr(), vh.data_ptr(), qh.data_ptr(), oh.data_ptr(), frames)
            assert rc == ckv.ERR_CUDA
            assert hio.counters() == before
            assert lib.convkv_attend_host(hio._h, qh.data_ptr(), oh.data_ptr()) == ckv.ERR_BAD_ORDER
            for j, (o_dev, (_, _, _, o)) in enumerate(zip(expected[:-1], queued)):
                assert np.array_equal(o_dev.view(torch.int16).cpu().numpy(), o.view(torch.int16).numpy()), j
        hio.step_host_async(kh, vh, qh, oh)
        queued.append((qh, kh, vh, oh))
    hio.sync()
    torch.cuda.synchronize()
    for i, (o_dev, (_, _, _, oh)) in enumerate(zip(expected, queued)):
        assert np.array_equal(o_dev.view(torch.int16).cpu().numpy(), oh.view(torch.int16).numpy()), i
    assert dev.counters() == hio.counters()
    assert dev.status() == 0 and hio.status() == 0
    dev.close()
    hio.close()

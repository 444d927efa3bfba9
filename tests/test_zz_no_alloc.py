"""The allocation-free e4m3 quantiser against the handle's own quantiser.

convkv_quantize_e4m3_noalloc serves callers that cannot allocate device memory
while they run (a serving engine handing out every device byte from its own
fixed pool, or a latency-critical thread where cudaMalloc would synchronise the
device).  Its scratch is a fixed array inside the library.  Here its codes and
scales are compared with those the fp8 append of a regular handle (the existing
entry points convkv_append_block + convkv_read_ring) writes for the same frames,
on two calls in a row, so a call that did not clear the shared scratch from the
previous one would show.  This file is collected last so that a failure here
comes after every other test has run; it also passes alone in a fresh process.
"""
from dataclasses import replace

import numpy as np
import pytest

import seeded_inputs as si
from compressed_kv_cache_convkv_b200.configs import PRESETS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    assert t.cuda.is_available(), "GPU tests need a CUDA device"
    from compressed_kv_cache_convkv_b200 import build
    build.build()
    si.build(device=True)
    return t


def _frames(t, w, tensor, frame0, n):
    x = t.empty((1, n * w.T, w.heads, w.head_dim), dtype=t.bfloat16, device="cuda")
    si.frames_device(x.data_ptr(), w.seed, tensor, 0, frame0, n, w.T * w.heads * w.head_dim, 1.0,
                     t.cuda.current_stream().cuda_stream)
    return x


@pytest.mark.parametrize("name", ["tiny", "fp8_480x832"])
def test_noalloc_quantiser_matches_append_quantiser_two_calls(torch, name):
    import compressed_kv_cache_convkv_b200 as ckv
    w = replace(PRESETS[name], fp8=True, num_states=1)
    b = w.block_frames
    cfg = w.config()
    wts = torch.zeros((1, 2, w.heads, w.head_dim, w.head_dim, 5), dtype=torch.bfloat16, device="cuda")
    h = ckv.ConvKV(cfg, wts)
    codes = torch.empty((b, w.T, w.heads, w.head_dim), dtype=torch.uint8, device="cuda")
    scales = torch.empty((b, w.heads), dtype=torch.float32, device="cuda")
    # warm-up: the first call on a device resolves the scratch array's address, and
    # the driver loads this part of the library's device code on first use
    ckv.quantize_e4m3_noalloc(torch.zeros((b, w.T, w.heads, w.head_dim), dtype=torch.bfloat16, device="cuda"),
                              codes, scales)
    torch.cuda.synchronize()
    F = 0
    for call in range(2):                      # two calls in a row, different frames
        k = _frames(torch, w, si.K, F, b)
        v = _frames(torch, w, si.V, F, b)
        h.append(k, v)                          # existing path: quantises k into the ring
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        codes.fill_(0xFF)                       # poison: every byte must be written
        scales.fill_(-1.0)
        torch.cuda.synchronize()
        ckv.quantize_e4m3_noalloc(k.view(b, w.T, w.heads, w.head_dim), codes, scales)
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0, "the call must not allocate device memory"
        got_c = codes.cpu().numpy()
        got_s = scales.cpu().numpy()
        for f in range(b):
            ref_c, ref_s = h.read_ring(0, 0, (F + f) % cfg.ring_frames)
            assert np.array_equal(got_c[f], ref_c), (name, call, f)
            assert np.array_equal(got_s[f], ref_s), (name, call, f)
        F += b
    h.close()


def test_noalloc_rejects_requests_beyond_the_scratch(torch):
    import compressed_kv_cache_convkv_b200 as ckv
    lib = ckv.library()
    x = torch.zeros((1, 8, 8), dtype=torch.bfloat16, device="cuda")
    c = torch.zeros((1, 8, 8), dtype=torch.uint8, device="cuda")
    s = torch.zeros((ckv.NOALLOC_MAX_FRAME_HEADS + 1,), dtype=torch.float32, device="cuda")
    rc = lib.convkv_quantize_e4m3_noalloc(x.data_ptr(), c.data_ptr(), s.data_ptr(), ckv.NOALLOC_MAX_FRAME_HEADS + 1,
                                          1, 1, 8, None)
    assert rc == ckv.ERR_SCRATCH_LIMIT
    assert lib.convkv_strerror(rc) == b"request exceeds the fixed scratch area"
    assert lib.convkv_quantize_e4m3_noalloc(None, c.data_ptr(), s.data_ptr(), 1, 1, 1, 8, None) == ckv.ERR_INVALID_ARG

"""bench.py on the host: the rank launcher, the algorithmic byte counts and the
reference arm (the oracle timed on a bounded sample), without a GPU."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from compressed_kv_cache_convkv_b200.configs import PRESETS  # noqa: E402


def test_gpus_n_starts_n_ranks_through_torchrun(monkeypatch):
    seen = {}
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(bench.subprocess, "call", lambda cmd: seen.setdefault("cmd", cmd) and 0)
    argv = ["--gpus", "4", "--steps", "2", "--warmup", "3", "--workload", "512x512"]
    assert bench.main(argv) == 0
    cmd = seen["cmd"]
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-len(argv):] == argv and cmd[-len(argv) - 1].endswith("bench.py")


def test_inside_torchrun_no_second_launch(monkeypatch):
    """Under torchrun (WORLD_SIZE set) the ranks run the workload themselves."""
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(bench.subprocess, "call", lambda cmd: pytest.fail("launched again"))
    monkeypatch.setattr(bench, "run_ours", lambda args, w: 7)
    assert bench.main(["--gpus", "2"]) == 7


def test_algorithmic_bytes():
    w = PRESETS["512x512"]
    fe = w.T * w.heads * w.head_dim
    # bf16: append reads K,V and writes K,V and the rotated K; one group reads 10 frames, writes 2
    wts = 2 * w.heads * 5 * w.head_dim ** 2 * 2
    assert bench.append_compress_bytes(w, 8, 1, 1.0) == 5 * 8 * fe * 2 + 12 * fe * 2 + wts
    f8 = PRESETS["fp8_480x832"]
    fe8 = f8.T * f8.heads * f8.head_dim
    wts8 = 2 * f8.heads * 5 * f8.head_dim ** 2 * 2
    assert bench.append_compress_bytes(f8, 8, 2, 2.0) == 2 * (2 * 8 * fe8 * 5 + 2 * (12 * fe8 + wts8))
    # attention: Q and O in bf16, K and V per key at the cache's width except bf16 keys
    assert bench.attention_bytes(10, 100, 128, 2) == (2 * 10 * 2 * 128 * 2 + 2 * 100 * 2 * 128 * 2)
    assert bench.attention_bytes(10, 100, 128, 2, kv_bytes=1.0, Nk_bf16=20) == \
        (2 * 10 * 2 * 128 * 2 + 2 * 20 * 2 * 128 * 2 + 2 * 80 * 2 * 128 * 1)


def test_reference_arm_prints_one_line(capsys):
    rc = bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3"])
    assert rc == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_peaks_fall_back_per_figure():
    """The measured peaks file may be absent, flat, nested or partial: each roofline
    denominator is the measured figure when one is found (any depth), else its
    fallback, and the source of each is reported."""
    fb = dict(bench.FALLBACK_PEAKS)
    pk, src = bench.parse_peaks(None)
    assert pk == fb and set(src.values()) == {"fallback"}
    pk, src = bench.parse_peaks({"hbm_gbs": 6543.4, "bf16_tflops": 1637.0, "bf16_tflops_sustained": 1386.2})
    assert pk == {"hbm_gbs": 6543.4, "bf16_tflops": 1637.0, "bf16_tflops_sustained": 1386.2}
    assert set(src.values()) == {"measured"}
    pk, src = bench.parse_peaks({"gpu": {"bf16_tflops": 1600}, "clocks": [1965], "hbm_gbs": "n/a"})
    assert pk["bf16_tflops"] == 1600.0 and src["bf16_tflops"] == "measured"
    assert pk["hbm_gbs"] == fb["hbm_gbs"] and src["hbm_gbs"] == "fallback"
    assert pk["bf16_tflops_sustained"] == fb["bf16_tflops_sustained"]
    pk, _ = bench.parse_peaks({"bf16_tflops": -1, "bf16_tflops_sustained": True})
    assert pk == fb

#!/usr/bin/env python
"""Benchmark of the ConvKV Memory attention step on B200.

One step = one block of the stream through the whole path: append (promote,
evict + conv-compress, ring copy or quantisation) and the fused reset-RoPE
attention, for every layer state of the workload.  The default workload is the
largest single-GPU one: 480x832 video (H=40, D=128, 30x52 tokens, blocks of 8
frames, window 10, memory 8) with the e4m3 K/V cache and 40 independent layer
states per call, in steady state (memory full), inputs resident in HBM.
--workload picks another preset (512x512, 720x416, nvfp4_480x832, ...).

Prints one JSON line (rank 0).  With --impl reference the fp64 CPU oracle is
timed instead, on a bounded sample of the same workload.  --gpus N without a
torchrun environment launches N ranks through torch.distributed.run; each rank
runs its own replica of the workload (independent layer states, no collective
on the data path) and rank 0 prints the max-over-ranks timing.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import socket
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ConvKV attend TFLOP/s (append+compress+attend step), latent frames/s per layer-step, % bf16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_BF16_TFLOPS = 2250.0   # B200 dense bf16, for context beside the measured peak
DEFAULT_WORKLOAD = "fp8_480x832"
CSRC = os.path.join(ROOT, "compressed_kv_cache_convkv_b200", "csrc")
# sources of the attend call, per cache format: the attention kernel, and in the
# e4m3 / NVFP4 formats the dequantisation that runs before it
ATTN_SOURCES = ("kernel_attn.cu", "sm100.cuh", "convkv_internal.h", "rope.cuh")
DEQUANT_SOURCES = ("kernels_dequant.cu", "lowp_codes.cuh", "nvfp4.cuh", "quant_div.cuh", "token_walk.h")


def attend_sources(fmt: str):
    return ATTN_SOURCES if fmt == "bf16" else ATTN_SOURCES + DEQUANT_SOURCES


def parse_peaks(d):
    """The roofline denominators from the measured peaks' JSON object: hbm_gbs,
    bf16_tflops and bf16_tflops_sustained found at any depth, each missing or unusable
    one replaced by its fallback.  Returns (peaks, {key: "measured" | "fallback"})."""
    out, src = dict(FALLBACK_PEAKS), {k: "fallback" for k in FALLBACK_PEAKS}

    def walk(x):
        if isinstance(x, dict):
            for k, v in x.items():
                if k in FALLBACK_PEAKS and src[k] == "fallback" and isinstance(v, (int, float)) \
                        and not isinstance(v, bool) and v > 0:
                    out[k], src[k] = float(v), "measured"
                else:
                    walk(v)
        elif isinstance(x, list):
            for v in x:
                walk(v)
    walk(d)
    return out, src


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p)) if os.path.exists(p) else None
    except (OSError, ValueError):
        d = None
    return parse_peaks(d)


def kv_format(w) -> str:
    return "nvfp4" if getattr(w, "fp4", False) else ("e4m3" if w.fp8 else "bf16")


def kv_bytes_per_value(w) -> float:
    """Cached K/V bytes per value: bf16 2, e4m3 1, NVFP4 1/2 + 1/16 (block scales)."""
    return {"bf16": 2.0, "e4m3": 1.0, "nvfp4": 9.0 / 16.0}[kv_format(w)]


def attention_flops(Nq, Nk, D, H, S=1):
    return 4.0 * Nq * Nk * D * H * S


def attention_bytes(Nq, Nk, D, H, S=1, kv_bytes=2.0, Nk_bf16=None):
    """Algorithmic HBM bytes of one attend: Q and O (bf16) plus every key's K and V, at
    kv_bytes per element, except the Nk_bf16 keys kept in bf16 (the current block and
    reference frames of the low-precision formats)."""
    nb = Nk if Nk_bf16 is None else Nk_bf16
    return (2.0 * Nq * H * D * 2 + 2.0 * nb * H * D * 2 + 2.0 * (Nk - nb) * H * D * kv_bytes) * S


def append_compress_bytes(w, b, S, groups_per_step, mean=False):
    """Algorithmic HBM bytes per step of append + compress.
    bf16: read the block's K and V, write them and the rotated K; per conv group read 5
    frames of K and V, write one slot of each, read both conv weights (none for the mean).
    e4m3 / NVFP4: read the block's K and V, write their bf16 staging copy and their codes
    (+ scales); per group read 5 frames of codes, write one slot of codes, read the weights."""
    fe = w.T * w.heads * w.head_dim                 # values per frame
    kvb = kv_bytes_per_value(w)
    weights = 0.0 if mean else 2.0 * w.heads * 5 * w.head_dim * w.head_dim * 2
    if kvb == 2.0:
        append = 5.0 * b * fe * 2
    else:
        append = 2.0 * b * fe * (2 + 2 + kvb)
    compress = groups_per_step * (12.0 * fe * kvb + weights)
    return S * (append + compress)


def source_sha(files) -> str:
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(CSRC, f), "rb").read())
    return h.hexdigest()


def measured_traffic(fmt: str, workload: str, algorithmic_bytes: float):
    """DRAM bytes per attention launch from the committed ncu capture of this kernel
    instantiation and workload (profiles/attn_kernel_<fmt>_<workload>.json), scaled to
    this launch's algorithmic bytes; None when there is none or the kernel sources
    changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"attn_kernel_{fmt}_{workload}.json")
    if not os.path.exists(path):
        return None, None
    d = json.load(open(path))
    if d.get("source_sha256") != source_sha(attend_sources(fmt)):
        return None, os.path.relpath(path, ROOT) + " (stale: kernel changed since the capture)"
    return (float(d["dram_bytes_per_launch"]) / float(d["algorithmic_bytes_per_launch"]) * algorithmic_bytes,
            os.path.relpath(path, ROOT))


# ----------------------------------------------------------------- CPU oracle

class OracleSample:
    """A steady-state oracle state of workload w (memory full, 8 window frames, one
    block), built directly from seeded frames for a subset of heads (heads are
    independent through the step), plus the block's queries.  In the e4m3 / NVFP4
    formats the memory and window frames hold their quantised values, as in the
    stream.  Setup (frame generation, quantisation) is not timed."""

    def __init__(self, w, heads):
        import numpy as np
        import seeded_inputs as si
        from oracle import convkv_oracle as O
        self.w, self.heads = w, list(heads)
        H = len(self.heads)
        cfg = O.OracleConfig(H=H, D=w.head_dim, grid_h=w.grid_h, grid_w=w.grid_w, window=w.window_frames,
                             mem_slots=w.mem_slots, fp8=w.fp8, fp4=getattr(w, "fp4", False))
        wts = si.bf16_bits_to_f64(si.conv_weights(w.seed, 0, w.heads, w.head_dim))[:, self.heads]
        st = O.OracleStream(cfg, wts)
        hs = np.asarray(self.heads)
        idx = ((np.arange(w.T)[:, None, None] * w.heads + hs[None, :, None]) * w.head_dim
               + np.arange(w.head_dim)[None, None, :]).reshape(-1)

        def fr(tensor, f):
            return si.bf16_bits_to_f64(si.frame_elements(w.seed, tensor, 0, f, idx)).reshape(w.T, H, w.head_dim)

        lowp = cfg.fp8 or cfg.fp4
        # memory slots are stored in the cache's type; window frames were quantised when
        # they joined the window (low-precision formats) or are the exact inputs (bf16)
        mem_value = (lambda x: st._quantize(x)[0]) if lowp else O.round_to_bf16
        win_value = (lambda x: st._quantize(x)[0]) if lowp else (lambda x: x)
        C, W, b = w.mem_slots, 8, w.block_frames
        st.memory = [O._Frame(mem_value(fr(si.K, 1000 + i)), mem_value(fr(si.V, 1000 + i)), i) for i in range(C)]
        st.window = [O._Frame(win_value(fr(si.K, 40 + i)), win_value(fr(si.V, 40 + i)), 40 + i) for i in range(W)]
        st.current = [O._Frame(fr(si.K, 48 + i), fr(si.V, 48 + i), 48 + i) for i in range(b)]
        self.st = st
        self.q = np.stack([fr(si.Q, 48 + i) for i in range(b)])
        self.group = np.stack([f.k for f in st.window[:5]])
        self.wk = wts[0]
        self.Nk = (C + W + b) * w.T
        self.Nq = b * w.T

    def time(self, rows: int, seed: int):
        """Seconds and algorithmic FLOPs of the oracle's attention on `rows` query rows
        (the sample's heads) plus one K conv group."""
        import numpy as np
        from oracle import convkv_oracle as O
        r = np.random.default_rng(seed).choice(self.Nq, size=min(rows, self.Nq), replace=False)
        t0 = time.perf_counter()
        self.st.attend(self.q, rows=r)
        O.conv_compress(self.group, self.wk)
        dt = time.perf_counter() - t0
        H, D = len(self.heads), self.w.head_dim
        conv = 2.0 * self.w.T * 5 * D * D * H
        return dt, attention_flops(len(r), self.Nk, D, H) + conv


SAMPLE_HEADS = (0, 5, 11, 17, 22, 28, 33, 39)


def cpu_baseline(w, rows: int = 4096):
    sample = OracleSample(w, [h for h in SAMPLE_HEADS if h < w.heads])
    dt, flops = sample.time(rows, 0)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{rows} query rows x {len(sample.heads)} heads of one steady-state {w.name} block "
                      f"({kv_format(w)} cache, Nk={sample.Nk}) + one conv group, fp64 numpy, {dt:.1f} s"}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    rows = 64
    sample = OracleSample(w, [h for h in SAMPLE_HEADS if h < w.heads])
    for i in range(args.warmup):
        sample.time(rows, 1000 + i)
    total_dt, total_flops = 0.0, 0.0
    for i in range(args.steps):
        dt, fl = sample.time(rows, i + 1)
        total_dt += dt
        total_flops += fl
    value = total_flops / total_dt / 1e12
    desc = (f"{rows} query rows x {len(sample.heads)} heads of a steady-state {w.name} block "
            f"({kv_format(w)} cache, Nk={sample.Nk}) + one conv group per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded Philox4x32-10, Irwin-Hall(12) unit-variance bf16 values)",
            "config": {"workload": f"{w.name} steady state, oracle sample: {desc}", "Nk": sample.Nk},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.file.flush()
        rows = []
        for line in open(self.file.name):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), float(f[3]), f[4], f[5:9]))
            except ValueError:
                continue
        os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        smax = max(r[1] for r in rows)
        loaded = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[4]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(loaded)}


# ----------------------------------------------------------------- our path

def run_ours(args, w):
    import torch
    import seeded_inputs as si
    import compressed_kv_cache_convkv_b200 as ckv
    from compressed_kv_cache_convkv_b200 import build
    from compressed_kv_cache_convkv_b200.sharding import max_over_ranks

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if rank == 0:
        build.build()
        si.build(device=True)
    if dist is not None:
        dist.barrier()

    S, H, D, T = w.num_states, w.heads, w.head_dim, w.T
    r = args.sink_frames
    mean = args.compress == "mean"
    fmt = kv_format(w)
    cfg = w.config(host_io=not args.no_e2e, sink_frames=r,
                   compress_mode=ckv.COMPRESS_MEAN if mean else ckv.COMPRESS_CONV)
    stream = torch.cuda.current_stream()
    fe = T * H * D
    # conv weights and inputs: seeded, generated on the device (each rank its own layer states)
    weights = torch.empty((S, 2, H, D, D, 5), dtype=torch.bfloat16, device="cuda")
    for s in range(S):
        for kv, tid in ((0, si.WK), (1, si.WV)):
            si.frames_device(weights[s, kv].data_ptr(), w.seed + rank, tid, s, 0, 1, H * D * D * 5,
                             si.weight_scale(D), stream.cuda_stream)
    h = ckv.ConvKV(cfg, None if mean else weights, stream=stream)
    del weights
    if r:
        # reference-image frames, attended first by every block
        ref = []
        for tid in (si.RK, si.RV):
            x = torch.empty((S, r * T, H, D), dtype=torch.bfloat16, device="cuda")
            for s in range(S):
                si.frames_device(x[s].data_ptr(), w.seed + rank, tid, s, 0, r, fe, 1.0, stream.cuda_stream)
            ref.append(x)
        h.set_sink(*ref)
    b = w.block_frames
    npool = 3
    pool = []
    for p in range(npool):
        t3 = []
        for tid in (si.Q, si.K, si.V):
            x = torch.empty((S, b * T, H, D), dtype=torch.bfloat16, device="cuda")
            for s in range(S):
                si.frames_device(x[s].data_ptr(), w.seed + rank, tid, s, 100 + p * b, b, fe, 1.0, stream.cuda_stream)
            t3.append(x)
        pool.append(t3)
    out = torch.empty((S, b * T, H, D), dtype=torch.bfloat16, device="cuda")

    def step(i):
        q, k, v = pool[i % npool]
        h.append(k, v)
        return q

    # fill to steady state (memory full) -- untimed
    first = w.first_block_frames
    q0, k0, v0 = (x[:, : first * T].contiguous() for x in pool[0])
    h.append(k0, v0)
    h.attend(q0)
    del q0, k0, v0
    while h.counters()["m"] < w.mem_slots or h.counters()["blocks"] < 8:
        q = step(0)
        h.attend(q, out)
    for i in range(args.warmup):
        q = step(i)
        h.attend(q, out)
    torch.cuda.synchronize()

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flops, nk_list = [], []
    groups = 0
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = h.launch_count()
    with ClockSampler(local) as clk:
        start.record(stream)
        for i in range(K):
            q = step(i)
            c = h.counters()
            groups += c["groups"]
            nk = (r + c["m"] + c["w"] + c["b"]) * T
            nk_list.append(nk)
            flops.append(attention_flops(b * T, nk, D, H, S))
            ev[i][0].record(stream)
            h.attend(q, out)
            ev[i][1].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
    launches = h.launch_count() - launches0
    total_ms = start.elapsed_time(end)
    att_ms = [a.elapsed_time(bb) for a, bb in ev]
    total_ms = max_over_ranks(total_ms, dist, "cuda")
    clocks = clk.summary()

    # end to end through the host-buffer entry points: pinned host q/k/v in, host out back, every step
    e2e_line = None
    if not args.no_e2e:
        # pinned host buffers, filled straight from the device; with several ranks on one
        # node, K and V share one buffer (the same bytes cross PCIe every step) so that
        # eight 40-state replicas stay well inside the host's memory
        def pinned_copy(x):
            hbuf = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
            hbuf.copy_(x)
            return hbuf
        qh = pinned_copy(pool[0][0])
        kh = pinned_copy(pool[0][1])
        vh = kh if world > 1 else pinned_copy(pool[0][2])
        oh = torch.empty(qh.shape, dtype=qh.dtype, pin_memory=True)
        Ke = max(3, min(K, 10))
        for _ in range(2):
            h.step_host(kh, vh, qh, oh)
        torch.cuda.synchronize()
        # the steps are queued back to back (convkv_step_host_async): a step's copies in
        # overlap the previous step's kernels; every step still copies its q, k, v in and
        # its outputs back; one sync at the end, before the closing event
        e2e_flops = 0.0
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist is not None:
            dist.barrier()
        e0.record(stream)
        for _ in range(Ke):
            # one pipelined call per step: append + attend from and to host buffers
            h.step_host_async(kh, vh, qh, oh)
            c = h.counters()
            e2e_flops += attention_flops(b * T, (r + c["m"] + c["w"] + c["b"]) * T, D, H, S)
        h.sync()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        e2e_ms = max_over_ranks(e2e_ms, dist, "cuda")
        e2e_line = {"value": e2e_flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": 3 * S * b * fe * 2, "d2h_bytes_per_step": S * b * fe * 2,
                    "steps": Ke, "ms_per_step": e2e_ms / Ke}
        del qh, kh, vh, oh
    assert h.status() == 0, "device status reported an error"

    pk, kind = peaks()
    total_flops = sum(flops) * world
    value = total_flops / (total_ms * 1e-3) / 1e12
    att_avg_ms = statistics.mean(att_ms)
    att_achieved = statistics.mean(flops) / (att_avg_ms * 1e-3) / 1e12
    # a kernel timed alone against the burst peak; one timed inside a seconds-long loop
    # (the 40-state workloads) against the sustained one, reached under the power cap
    sustained = total_ms > 1000.0
    pkey = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    peak = pk[pkey]
    kvb = kv_bytes_per_value(w)
    att_bytes = attention_bytes(b * T, statistics.mean(nk_list), D, H, S, kv_bytes=kvb,
                                Nk_bf16=(b + r) * T if kvb < 2 else None)
    traffic, traffic_src = measured_traffic(fmt, w.name, att_bytes)
    frames_per_s = K * b * S * world / (total_ms * 1e-3)
    ac_ms = (total_ms - sum(att_ms)) / K
    ac_line = None
    if ac_ms > 0:
        acb = append_compress_bytes(w, b, S, groups / K, mean=mean)
        ac_line = {"bytes_per_step": acb, "gbs": acb / (ac_ms * 1e-3) / 1e9,
                   "frac_of_hbm": acb / (ac_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                   "note": "event time between attends: append, conv groups, the time-table copy and launch gaps"}
    kernel = ("attn_kernel<128>" if fmt == "bf16" else
              "attn_kernel<128> with dequant_kernel<128> before it (the attend call: the e4m3 / NVFP4 "
              "window and memory dequantised once per attend into a bf16 scratch)")
    dtype = {"bf16": "bf16", "e4m3": "bf16 compute, e4m3 K/V cache", "nvfp4": "bf16 compute, NVFP4 K/V cache"}[fmt]
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": dtype, "data": "synthetic (seeded Philox4x32-10, Irwin-Hall(12) unit-variance bf16 values)",
        "config": {"workload": f"{w.name} steady state (memory full), {S} layer state(s) per GPU"
                               + (f", {r} reference-image frame(s) attended first" if r else "")
                               + (", mean memory (5-frame mean instead of the conv)" if mean else ""),
                   "preset": w.name, "kv_format": fmt,
                   "heads": H, "head_dim": D, "tokens_per_frame": T, "block_frames": b,
                   "window_frames": w.window_frames, "mem_slots": w.mem_slots, "reference_frames": r,
                   "compress": args.compress, "states": S,
                   "keys_per_step_avg": statistics.mean(nk_list), "state_bytes": h.state_bytes(),
                   "l2": f"inputs larger than L2 (q,k,v {3 * S * b * fe * 2 / 1e6:.0f} MB/step + "
                         f"{h.state_bytes() / 1e6:.0f} MB cache state vs 126 MB L2)",
                   "parallelism": f"replicas x{world} (independent layer states, no collective)"},
        "latent_frames_per_s_per_layer_step": frames_per_s,
        "pct_bf16_peak": 100.0 * value / peak,
        "kernels_ms": {"attend_avg": att_avg_ms, "append_compress_avg": ac_ms,
                       "conv_groups_per_step": groups / K},
        "append_compress": ac_line,
        "pct_of_spec_bf16_2250": 100.0 * att_achieved / SPEC_BF16_TFLOPS,
        "roofline": {"bound": "tensor", "achieved": att_achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": att_achieved / peak, "traffic": traffic,
                     "algorithmic_bytes": att_bytes, "kernel": kernel,
                     "peak_source": (f"measured bf16 {'sustained' if sustained else 'burst'} (MEASURED_PEAKS.json)"
                                     if kind[pkey] == "measured" else
                                     f"fallback bf16 {'sustained' if sustained else 'burst'} ({peak:.0f} TF/s, "
                                     "earlier measurement on this pool; no such figure in MEASURED_PEAKS.json "
                                     "on the box)"),
                     "frac_of_burst": att_achieved / pk["bf16_tflops"],
                     "traffic_source": traffic_src},
        "e2e": e2e_line,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    h.close()
    del pool, out
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- launcher

def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def rank_launch_command(n: int, argv) -> list:
    """torch.distributed.run command that starts n ranks of this script on one node."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
            os.path.abspath(__file__)] + list(argv)


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--compress", choices=["conv", "mean"], default="conv",
                    help="memory compression: the learned 1D conv (default) or the 5-frame mean")
    ap.add_argument("--sink-frames", type=int, default=0,
                    help="reference-image frames attended first by every block (default none)")
    ap.add_argument("--states", type=int, default=0,
                    help="layer states per call (default: the workload's own; fewer make a small profiling case)")
    args = ap.parse_args(argv)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start the ranks here and pass their output through
        return subprocess.call(rank_launch_command(args.gpus, argv))
    from dataclasses import replace
    from compressed_kv_cache_convkv_b200.configs import PRESETS
    w = PRESETS[args.workload]
    if args.states:
        w = replace(w, num_states=args.states)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())

#!/usr/bin/env python
"""Benchmark of the ConvKV Memory attention step on B200.

One step = one block of the stream through the whole path: append (promote,
evict + conv-compress, ring copy) and the fused reset-RoPE attention.  The
workload is the 512x512 shape (H=40, D=128, 32x32 tokens, blocks of 8 frames,
window 10, memory 8) in steady state (memory full), inputs resident in HBM.

Prints one JSON line (rank 0).  With --impl reference the fp64 CPU oracle is
timed instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
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


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def attention_flops(Nq, Nk, D, H, S=1):
    return 4.0 * Nq * Nk * D * H * S


def attention_bytes(Nq, Nk, D, H, S=1, kv_bytes=2, Nk_bf16=None):
    """Algorithmic HBM bytes of one attend: Q and O (bf16) plus every key's K and V, at
    kv_bytes per element (e4m3 1, NVFP4 9/16 with its block scales) except the Nk_bf16
    keys kept in bf16 (the current block and reference frames of the low-precision formats)."""
    nb = Nk if Nk_bf16 is None else Nk_bf16
    return (2.0 * Nq * H * D * 2 + 2.0 * nb * H * D * 2 + 2.0 * (Nk - nb) * H * D * kv_bytes) * S


def measured_traffic(algorithmic_bytes):
    """DRAM bytes per attention launch from the committed ncu capture, scaled to this
    launch's algorithmic bytes; None when the kernel sources changed since the capture."""
    import hashlib
    prof = os.path.join(ROOT, "profiles", "attn_kernel_512x512.md")
    src = os.path.join(ROOT, "compressed_kv_cache_convkv_b200", "csrc")
    if not os.path.exists(prof):
        return None
    fields = {}
    for line in open(prof):
        if ":" in line and line.split(":")[0] in ("source_sha256", "dram_bytes_per_launch",
                                                  "algorithmic_bytes_per_launch"):
            k, v = line.split(":", 1)
            fields[k] = v.strip()
    h = hashlib.sha256()
    for f in ("kernel_attn.cu", "sm100.cuh", "convkv_internal.h"):
        h.update(open(os.path.join(src, f), "rb").read())
    if fields.get("source_sha256") != h.hexdigest():
        return None
    return float(fields["dram_bytes_per_launch"]) / float(fields["algorithmic_bytes_per_launch"]) * algorithmic_bytes


# ----------------------------------------------------------------- CPU oracle

def oracle_sample(w, rows: int, seed_offset: int = 0):
    """A steady-state oracle state of workload w built directly from seeded frames
    (memory slots, window, current block), plus the queries of the current block."""
    import numpy as np
    import seeded_inputs as si
    from oracle import convkv_oracle as O
    cfg = O.OracleConfig(H=w.heads, D=w.head_dim, grid_h=w.grid_h, grid_w=w.grid_w, window=w.window_frames,
                         mem_slots=w.mem_slots)
    wts = si.bf16_bits_to_f64(si.conv_weights(w.seed, 0, w.heads, w.head_dim))
    st = O.OracleStream(cfg, wts)
    fe = w.T * w.heads * w.head_dim
    shape = (w.T, w.heads, w.head_dim)

    def fr(tensor, f):
        return si.bf16_bits_to_f64(si.frames(w.seed, tensor, 0, f, 1, fe)).reshape(shape)

    C, W, b = w.mem_slots, 8, w.block_frames
    st.memory = [O._Frame(O.round_to_bf16(fr(si.K, 1000 + i)), O.round_to_bf16(fr(si.V, 1000 + i)), i)
                 for i in range(C)]
    st.window = [O._Frame(fr(si.K, 40 + i), fr(si.V, 40 + i), 40 + i) for i in range(W)]
    st.current = [O._Frame(fr(si.K, 48 + i), fr(si.V, 48 + i), 48 + i) for i in range(b)]
    q = np.stack([fr(si.Q, 48 + i) for i in range(b)])
    group = np.stack([fr(si.K, 40 + i) for i in range(5)])
    rng = np.random.default_rng(seed_offset)
    r = rng.choice(b * w.T, size=rows, replace=False)
    Nk = (C + W + b) * w.T
    return st, q, r, group, wts, Nk


def time_oracle(w, rows: int, reps: int = 1, seed_offset: int = 0):
    """Seconds and algorithmic FLOPs of the oracle on `rows` query rows (all heads) + one conv group."""
    from oracle import convkv_oracle as O
    st, q, r, group, wts, Nk = oracle_sample(w, rows, seed_offset)
    t0 = time.perf_counter()
    for _ in range(reps):
        st.attend(q, rows=r)
        O.conv_compress(group, wts[0])
    dt = time.perf_counter() - t0
    conv = 2.0 * w.T * 5 * w.head_dim * w.head_dim * w.heads
    flops = reps * (attention_flops(rows, Nk, w.head_dim, w.heads) + conv)
    return dt, flops, Nk


def append_compress_bytes(w, b, S, groups_per_step, mean=False):
    """Algorithmic HBM bytes per step of append + compress in the bf16 format: read the
    block's K and V, write them and the rotated K; per conv group read 5 frames of K and
    V, write one slot of each, read the conv weights of both (none for the mean)."""
    fb = w.T * w.heads * w.head_dim * 2                   # bytes of one bf16 frame
    append = 5.0 * S * b * fb
    weights = 0.0 if mean else 2.0 * w.heads * 5 * w.head_dim * w.head_dim * 2
    compress = groups_per_step * S * (12.0 * fb + weights)
    return append + compress


def cpu_baseline(w, budget_rows: int = 768):
    dt, flops, Nk = time_oracle(w, budget_rows)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{budget_rows} query rows x {w.heads} heads of one steady-state {w.name} block "
                      f"(Nk={Nk}) + one conv group, fp64 numpy, {dt:.1f} s"}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    rows = 32
    for _ in range(args.warmup):
        time_oracle(w, rows)
    total_dt, total_flops = 0.0, 0.0
    for i in range(args.steps):
        dt, fl, Nk = time_oracle(w, rows, seed_offset=i + 1)
        total_dt += dt
        total_flops += fl
    value = total_flops / total_dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded Philox4x32-10, Irwin-Hall(12) unit-variance bf16 values)",
            "config": {"workload": f"{w.name} steady state, oracle sample of {rows} query rows x {w.heads} heads "
                                   f"per step + one conv group", "Nk": Nk},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                             "sample": f"{rows} query rows x {w.heads} heads + one K conv group per step"},
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
    cfg = w.config(host_io=not args.no_e2e, sink_frames=r,
                   compress_mode=ckv.COMPRESS_MEAN if mean else ckv.COMPRESS_CONV)
    stream = torch.cuda.current_stream()
    fe = T * H * D
    # conv weights and inputs: seeded, generated on the device (each rank its own layer state)
    weights = torch.empty((S, 2, H, D, D, 5), dtype=torch.bfloat16, device="cuda")
    for s in range(S):
        for kv, tid in ((0, si.WK), (1, si.WV)):
            si.frames_device(weights[s, kv].data_ptr(), w.seed + rank, tid, s, 0, 1, H * D * D * 5,
                             si.weight_scale(D), stream.cuda_stream)
    h = ckv.ConvKV(cfg, None if mean else weights, stream=stream)
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
        qh = pool[0][0].cpu().pin_memory()
        kh = pool[0][1].cpu().pin_memory()
        vh = pool[0][2].cpu().pin_memory()
        oh = torch.empty_like(qh).pin_memory()
        Ke = max(3, min(K, 10))
        for _ in range(2):
            h.append_host(kh, vh)
            h.attend_host(qh, oh)
        torch.cuda.synchronize()
        e2e_flops = 0.0
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist is not None:
            dist.barrier()
        e0.record(stream)
        for _ in range(Ke):
            h.append_host(kh, vh)
            c = h.counters()
            e2e_flops += attention_flops(b * T, (r + c["m"] + c["w"] + c["b"]) * T, D, H, S)
            h.attend_host(qh, oh)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        e2e_ms = max_over_ranks(e2e_ms, dist, "cuda")
        e2e_line = {"value": e2e_flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": 3 * S * b * fe * 2, "d2h_bytes_per_step": S * b * fe * 2}
    assert h.status() == 0, "device status reported an error"

    pk, kind = peaks()
    total_flops = sum(flops) * world
    value = total_flops / (total_ms * 1e-3) / 1e12
    att_avg_ms = statistics.mean(att_ms)
    att_achieved = statistics.mean(flops) / (att_avg_ms * 1e-3) / 1e12
    peak = pk["bf16_tflops"]
    kvb = 9.0 / 16.0 if getattr(w, "fp4", False) else (1.0 if w.fp8 else 2.0)
    att_bytes = attention_bytes(b * T, statistics.mean(nk_list), D, H, S, kv_bytes=kvb,
                                Nk_bf16=(b + r) * T if kvb < 2 else None)
    # the committed capture is of the bf16 instantiation; other formats run another kernel
    traffic = measured_traffic(att_bytes) if kvb == 2.0 else None
    frames_per_s = K * b * S * world / (total_ms * 1e-3)
    ac_ms = (total_ms - sum(att_ms)) / K
    ac_line = None
    if kvb == 2.0 and ac_ms > 0:
        acb = append_compress_bytes(w, b, S, groups / K, mean=mean)
        ac_line = {"bytes_per_step": acb, "gbs": acb / (ac_ms * 1e-3) / 1e9,
                   "frac_of_hbm": acb / (ac_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                   "note": "event time between attends: append, conv groups, the time-table copy and launch gaps"}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if not w.fp8 and not getattr(w, "fp4", False) else
                 ("bf16 compute, e4m3 K/V cache" if w.fp8 else "bf16 compute, NVFP4 K/V cache"), "data": "synthetic (seeded Philox4x32-10, Irwin-Hall(12) unit-variance bf16 values)",
        "config": {"workload": f"{w.name} steady state (memory full), one layer state per GPU"
                               + (f", {r} reference-image frame(s) attended first" if r else "")
                               + (", mean memory (5-frame mean instead of the conv)" if mean else ""),
                   "heads": H, "head_dim": D, "tokens_per_frame": T, "block_frames": b,
                   "window_frames": w.window_frames, "mem_slots": w.mem_slots, "reference_frames": r, "compress": args.compress, "states": S,
                   "keys_per_step_avg": statistics.mean(nk_list), "state_bytes": h.state_bytes(),
                   "l2": f"inputs larger than L2 (q,k,v {3 * S * b * fe * 2 / 1e6:.0f} MB/step + "
                         f"{h.state_bytes() / 1e6:.0f} MB cache state vs 126 MB L2)",
                   "parallelism": f"replicas x{world} (independent layer states, no collective)"},
        "latent_frames_per_s_per_layer_step": frames_per_s,
        "pct_bf16_peak": 100.0 * value / peak,
        "kernels_ms": {"attend_avg": att_avg_ms, "append_compress_avg": (total_ms - sum(att_ms)) / K,
                       "conv_groups_per_step": groups / K},
        "append_compress": ac_line,
        "pct_of_spec_bf16_2250": 100.0 * att_achieved / SPEC_BF16_TFLOPS,
        "roofline": {"bound": "tensor", "achieved": att_achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": att_achieved / peak, "traffic": traffic,
                     "algorithmic_bytes": att_bytes, "kernel": "attn_kernel<128>",
                     "peak_source": f"{kind} bf16 burst (MEASURED_PEAKS.json)",
                     "traffic_source": "ncu dram__bytes_read+write of one launch (profiles/attn_kernel_512x512.md), "
                                       "scaled by algorithmic bytes; null if the kernel changed since"},
        "e2e": e2e_line,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    h.close()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="512x512")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer end-to-end leg (large multi-state workloads)")
    ap.add_argument("--compress", choices=["conv", "mean"], default="conv",
                    help="memory compression: the learned 1D conv (default) or the 5-frame mean")
    ap.add_argument("--sink-frames", type=int, default=0,
                    help="reference-image frames attended first by every block (default none)")
    args = ap.parse_args()
    from compressed_kv_cache_convkv_b200.configs import PRESETS
    w = PRESETS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())

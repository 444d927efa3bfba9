"""Sequence-parallel exchange on CPU: two gloo ranks, the fp64 oracle as the compute.

Each rank holds a sequence shard (every head) of each block of the tiny stream.  An
all-to-all turns the shards into head shards (all rows, this rank's heads), the
oracle runs the ConvKV step on those heads, and the inverse all-to-all returns each
rank's rows.  The result must equal the all-heads oracle on the rank's rows: this
pins the row split and head ownership rules the library's fused kernels implement
(shard_rows, head_range) and the reading that heads are independent in this step.
"""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

from compressed_kv_cache_convkv_b200.sp import head_range, shard_rows


def test_shard_rows_rule():
    for rows in (16, 32, 7020, 9360, 6144):
        for G in (1, 2, 3, 4, 8):
            off = shard_rows(rows, G)
            assert off[0] == 0 and off[-1] == rows and len(off) == G + 1
            sizes = np.diff(off)
            assert sizes.min() >= rows // G and sizes.max() <= rows // G + 1
    assert list(head_range(40, 8, 3)) == [15, 16, 17, 18, 19]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _all_to_all(dist, recv, send, rank):
    """recv[r] <- rank r's send[rank], by point-to-point messages (gloo has no all-to-all)."""
    reqs = []
    for r in range(len(send)):
        if r == rank:
            recv[r].copy_(send[r])
        else:
            reqs.append(dist.isend(send[r], r))
            reqs.append(dist.irecv(recv[r], r))
    for x in reqs:
        x.wait()


def _worker(rank, world, port, q):
    try:
        _work(rank, world, port, q)
    except Exception as e:  # report instead of leaving the parent waiting
        q.put((rank, repr(e)))
        raise


def _work(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import seeded_inputs as si
        from compressed_kv_cache_convkv_b200.configs import PRESETS
        from oracle import convkv_oracle as O
        w = PRESETS["tiny"]
        H, D, T = w.heads, w.head_dim, w.T
        wts = si.bf16_bits_to_f64(si.conv_weights(w.seed, 0, H, D))
        mine = head_range(H, world, rank)
        cfg = O.OracleConfig(H=len(mine), D=D, grid_h=w.grid_h, grid_w=w.grid_w, window=w.window_frames,
                             mem_slots=w.mem_slots)
        part = O.OracleStream(cfg, wts[:, mine.start:mine.stop])
        full = O.OracleStream(O.OracleConfig(H=H, D=D, grid_h=w.grid_h, grid_w=w.grid_w,
                                             window=w.window_frames, mem_slots=w.mem_slots), wts)
        F, worst = 0, 0.0
        for b in w.block_sizes():
            rows = b * T
            off = shard_rows(rows, world)
            blk = {t: si.bf16_bits_to_f64(si.frames(w.seed, t, 0, F, b, T * H * D)).reshape(rows, H, D)
                   for t in (si.Q, si.K, si.V)}
            shard = {t: torch.from_numpy(x[off[rank]:off[rank + 1]].copy()) for t, x in blk.items()}
            # sequence shard -> head shard
            got = {}
            for t, x in shard.items():
                send = [x[:, head_range(H, world, g).start:head_range(H, world, g).stop].contiguous()
                        for g in range(world)]
                recv = [torch.empty((off[r + 1] - off[r], len(mine), D), dtype=torch.float64) for r in range(world)]
                _all_to_all(dist, recv, send, rank)
                got[t] = torch.cat(recv).numpy().reshape(b, T, len(mine), D)
            part.append(got[si.K], got[si.V])
            o, _ = part.attend(got[si.Q])                       # [rows, my heads, D]
            # head shard -> sequence shard
            o = torch.from_numpy(np.ascontiguousarray(o.reshape(rows, len(mine), D)))
            send = [o[off[r]:off[r + 1]].contiguous() for r in range(world)]
            recv = [torch.empty((off[rank + 1] - off[rank], len(head_range(H, world, g)), D), dtype=torch.float64)
                    for g in range(world)]
            _all_to_all(dist, recv, send, rank)
            mine_out = torch.cat(recv, dim=1).numpy()           # my rows, every head
            full.append(blk[si.K].reshape(b, T, H, D), blk[si.V].reshape(b, T, H, D))
            ref, _ = full.attend(blk[si.Q].reshape(b, T, H, D))
            ref = ref.reshape(rows, H, D)[off[rank]:off[rank + 1]]
            worst = max(worst, float(np.abs(mine_out - ref).max()))
            F += b
        q.put((rank, worst))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_sequence_to_head_exchange_matches_all_heads():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, worst in res:
        assert isinstance(worst, float), (rank, worst)
        assert worst <= 1e-12, (rank, worst)

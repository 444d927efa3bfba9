"""Sequence-parallel use of the ConvKV step (one process per GPU).

SoulX-LiveAct runs its DiT with two-GPU sequence parallelism (blog walk-through,
system-level optimisation section, item (2)).  The activations entering this step
are then split by sequence: rank r holds rows [off_r, off_{r+1}) of the block's
frames*T rows, with every head.  Heads are independent in this step, so each
rank keeps the cache of its own H/G heads, and the exchange between the two
layouts (the all-to-all of q, k, v and its inverse on the output) is fused into
the library's kernels: convkv_append_block_sp and convkv_attend_sp read the
other ranks' shards and write the outputs back into them directly, through
pointers to peer memory.

This module holds the host side: the row split (the same rule as the library's),
the views of a block as shards, and, for a multi-GPU node, the exchange of the
shard buffers' CUDA IPC handles and the ordering of the ranks around each step.
"""
from __future__ import annotations

import ctypes
from typing import List, Sequence


def shard_rows(rows: int, ranks: int) -> List[int]:
    """Row offsets of the sequence shards: rank r holds rows [off[r], off[r+1]),
    off[r] = floor(r * rows / ranks) (the library's rule)."""
    if ranks < 1:
        raise ValueError("ranks must be >= 1")
    return [r * rows // ranks for r in range(ranks + 1)]


def split_block(x, ranks: int):
    """Views of a block [S, rows, heads, D] as its `ranks` sequence shards."""
    off = shard_rows(x.shape[1], ranks)
    return [x[:, off[r]:off[r + 1]] for r in range(ranks)]


def head_range(heads_total: int, ranks: int, rank: int) -> range:
    """Heads owned by `rank` (contiguous, heads_total / ranks each)."""
    if heads_total % ranks:
        raise ValueError(f"{heads_total} heads do not split over {ranks} ranks")
    n = heads_total // ranks
    return range(rank * n, (rank + 1) * n)


class SequenceParallelConvKV:
    """One rank of a G-rank group on a multi-GPU node.

    The rank owns the cache of heads head_range(H, G, rank) and four shard buffers
    (q, k, v, out) of [S, rows_max, H, D] bf16 that every rank maps by CUDA IPC.
    Per block: the caller writes its q/k/v rows into `shard(which)`, calls step(),
    and reads its output rows from `shard("out")`.  step() orders the ranks with
    two barriers of the process group: all shards are written before any rank's
    kernels read them, and all outputs are written before any rank reads its own.
    """

    WHICH = ("q", "k", "v", "out")

    def __init__(self, cfg, conv_weight, group=None):
        import torch
        import torch.distributed as dist
        from . import ConvKV, _lib
        self.dist, self.group = dist, group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        H = cfg.heads
        heads = head_range(H, self.G, self.rank)
        self.cfg = cfg.with_(heads=len(heads), sp_ranks=self.G, sp_rank=self.rank)
        w = conv_weight[:, :, heads.start:heads.stop].contiguous() if conv_weight is not None else None
        self.cache = ConvKV(self.cfg, w)
        rows_max = -(-cfg.max_block * cfg.T // self.G)
        self.bufs = {n: torch.zeros((cfg.num_states, rows_max, H, cfg.head_dim), dtype=torch.bfloat16,
                                    device="cuda") for n in self.WHICH}
        lib = _lib()
        mine = []
        for n in self.WHICH:
            handle = (ctypes.c_uint8 * 64)()
            offset = ctypes.c_size_t()
            rc = lib.convkv_ipc_export(self.bufs[n].data_ptr(), handle, ctypes.byref(offset))
            if rc:
                raise RuntimeError(f"convkv_ipc_export failed ({rc})")
            mine.append((bytes(handle), offset.value))
        everyone: list = [None] * self.G
        dist.all_gather_object(everyone, mine, group=group)
        self._opened = []
        self.peer = {n: [0] * self.G for n in self.WHICH}
        for r in range(self.G):
            for i, n in enumerate(self.WHICH):
                if r == self.rank:
                    self.peer[n][r] = self.bufs[n].data_ptr()
                    continue
                handle, offset = everyone[r][i]
                base = ctypes.c_void_p()
                rc = lib.convkv_ipc_open((ctypes.c_uint8 * 64).from_buffer_copy(handle), ctypes.byref(base))
                if rc:
                    raise RuntimeError(f"convkv_ipc_open of rank {r}'s {n} shard failed ({rc})")
                self._opened.append(base.value)
                self.peer[n][r] = base.value + offset

    def shard(self, which: str, frames: int):
        """This rank's rows of the block in buffer `which` ([S, rows_r, H, D])."""
        off = shard_rows(frames * self.cfg.T, self.G)
        return self.bufs[which][:, : off[self.rank + 1] - off[self.rank]]

    def step(self, frames: int) -> None:
        from . import _lib
        arr = lambda n: (ctypes.c_void_p * self.G)(*self.peer[n])
        self.dist.barrier(group=self.group)
        lib = _lib()
        rc = lib.convkv_append_block_sp(self.cache._h, arr("k"), arr("v"), frames)
        if rc == 0:
            rc = lib.convkv_attend_sp(self.cache._h, arr("q"), arr("out"))
        self.dist.barrier(group=self.group)
        if rc:
            raise RuntimeError(f"sequence-parallel step failed ({rc})")

    def close(self) -> None:
        from . import _lib
        for p in self._opened:
            _lib().convkv_ipc_close(ctypes.c_void_p(p))
        self._opened = []
        self.cache.close()

"""The five workloads the path is measured and checked on.

Shapes follow the Wan2.1-lineage DiT of SoulX-LiveAct (40 heads of 128
channels; blocks of 6 then 8 latent frames, SoulX-LiveAct blog walk-through,
"Neighbor Forcing" and Table 5 of the arXiv page).  Token grids are the latent
grids of the stated video sizes after the 2x2 patchify.  Inputs are seeded
synthetic bf16 values of unit variance.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List


@dataclass(frozen=True)
class Workload:
    name: str
    heads: int
    head_dim: int
    grid_h: int
    grid_w: int
    first_block_frames: int
    block_frames: int
    window_frames: int
    mem_slots: int
    stream_frames: int
    seed: int
    fp8: bool = False
    num_states: int = 1
    fp4: bool = False        # NVFP4 ring and memory

    @property
    def T(self) -> int:
        return self.grid_h * self.grid_w

    def block_sizes(self) -> List[int]:
        """Frames per block over the stream; the last block is short when the stream does not divide."""
        sizes = [self.first_block_frames]
        while sum(sizes) + self.block_frames <= self.stream_frames:
            sizes.append(self.block_frames)
        rest = self.stream_frames - sum(sizes)
        if rest > 0:
            sizes.append(rest)
        return sizes

    def config(self, **kw):
        from . import Config, KV_BF16, KV_FP8_E4M3, KV_NVFP4
        fmt = KV_NVFP4 if self.fp4 else (KV_FP8_E4M3 if self.fp8 else KV_BF16)
        c = Config(heads=self.heads, head_dim=self.head_dim, grid_h=self.grid_h, grid_w=self.grid_w,
                   first_block_frames=self.first_block_frames, block_frames=self.block_frames,
                   window_frames=self.window_frames, mem_slots=self.mem_slots,
                   kv_format=fmt, num_states=self.num_states)
        return c.with_(**kw) if kw else c


PRESETS = {
    # H=2, D=64, 4x4 tokens, blocks of 2, window 4, memory 3, 30 frames (15 blocks)
    "tiny": Workload("tiny", 2, 64, 4, 4, 2, 2, 4, 3, 30, seed=0),
    # 512x512 video: 32x32 tokens per latent frame, memory 8, 200 frames (26 blocks, last one 2 frames)
    "512x512": Workload("512x512", 40, 128, 32, 32, 6, 8, 10, 8, 200, seed=1),
    # 720x416 video: 45x26 = 1170 tokens (ragged tiles), memory 16, 300 frames (38 blocks)
    "720x416": Workload("720x416", 40, 128, 45, 26, 6, 8, 10, 16, 300, seed=2),
    # the 512x512 shape streamed for 18,000 latent frames (~72k video frames, 2,251 blocks)
    "soak": Workload("soak", 40, 128, 32, 32, 6, 8, 10, 8, 18000, seed=3),
    # fp8 e4m3 window/memory at 480x832: 30x52 = 1560 tokens, blocks of 8, 40 states per call
    "fp8_480x832": Workload("fp8_480x832", 40, 128, 30, 52, 8, 8, 10, 8, 200, seed=4, fp8=True, num_states=40),
    # the same shape with the NVFP4 window and memory (FP4 for B-series GPUs)
    "nvfp4_480x832": Workload("nvfp4_480x832", 40, 128, 30, 52, 8, 8, 10, 8, 200, seed=5, num_states=40, fp4=True),
}

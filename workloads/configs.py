"""Workload shapes for the DualParal window step (pure data, no arithmetic of the method).

Shapes follow the arXiv 2505.21070 pages ("Minute-Long Videos with Dual
Parallelisms", abstract: block-wise queue of frame blocks, feature cache of the
block that left) plus the five workload definitions this library is measured on:

* ``tiny_f32``      2 blocks x 128 tokens, 128-token cache, 2x64 heads, fp32.
* ``cogvideo_bf16`` 4 blocks x 2 latent frames x 1350 tokens (480x720 video, 8x VAE,
                    patch 2), 2700-token cache, 48x64 heads, bf16.
* ``wan_bf16``      8 blocks x 4 latent frames x 1560 tokens (832x480), 6240-token
                    cache, 12x128 heads, bf16.
* ``long_run``      257 latent frames x 1350 tokens in 2-frame blocks, window of 8
                    blocks, 50 staggered timesteps per block, 24x64 heads, bf16.
* ``longrun_steady_bf16``  one window step of the long run's steady state: 8 blocks x
                    2700 tokens, 2700-token cache, 24x64 heads, N(0,1) inputs.
* ``wan_paper_bf16`` the pages' own block size on the Wan-like latent: 4 blocks of 8 latent
                    frames x 1560 tokens, a cache of 8 latent frames (one exited block),
                    12x128 heads, bf16.
* ``sweep``         window of 4 blocks, 4096..131072 tokens, cache = window/4,
                    16x128 heads, bf16, with a ragged last block variant.

Rows of every token tensor are ordered head (cleanest block, smallest timestep)
first; the channel index is ``h * head_dim + d``.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

SEED_BASE = 20250527

CONFIG_NAMES = ["tiny_f32", "cogvideo_bf16", "wan_bf16", "long_run", "longrun_steady_bf16", "wan_paper_bf16", "sweep"]


@dataclass
class StepConfig:
    """One window step: a window of blocks, a one-block feature cache, a push."""
    name: str
    dtype: str                  # "f32" or "bf16"
    n_heads: int
    head_dim: int
    block_rows: List[int]       # rows per block, head block first
    cache_len: int              # valid cached rows at the start of the step
    cache_capacity: int         # rows the cache slot can hold
    timesteps: List[int]        # per block, head first (index into the 1000-row table)
    qkv_std: float              # std of the synthetic q, k, v, cache entries
    seed: int
    push_rows: int              # rows of the fresh noise block pushed by the advance
    table_rows: int = 1000      # adaLN table rows (one per diffusion timestep)
    random_timesteps: bool = False  # draw timesteps U{0..999} from the generator
    note: str = ""

    @property
    def hidden(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def n_win(self) -> int:
        return sum(self.block_rows)

    @property
    def n_blocks(self) -> int:
        return len(self.block_rows)

    @property
    def row_offset(self) -> List[int]:
        out = [0]
        for r in self.block_rows:
            out.append(out[-1] + r)
        return out

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def attn_flop(self) -> int:
        """QK^T plus PV multiply-adds (2 flop each) over valid rows only."""
        return 4 * self.n_win * (self.cache_len + self.n_win) * self.head_dim * self.n_heads


@dataclass
class RunConfig:
    """The full long-video queue run (every step until all blocks have exited)."""
    name: str
    n_heads: int
    head_dim: int
    n_frames: int
    frame_rows: int
    frames_per_block: int
    window_blocks: int          # W: blocks in the steady-state window
    n_timesteps: int            # T: evaluations per block
    seed: int
    table_rows: int = 1000

    @property
    def hidden(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def block_rows(self) -> List[int]:
        full, rest = divmod(self.n_frames, self.frames_per_block)
        rows = [self.frames_per_block * self.frame_rows] * full
        if rest:
            rows.append(rest * self.frame_rows)
        return rows

    @property
    def slot_rows(self) -> int:
        return self.frames_per_block * self.frame_rows


def _even_timesteps(n: int) -> List[int]:
    # evenly spaced in [0, 999], head (cleanest) first, rounded half-to-even
    if n == 1:
        return [0]
    return [int(round(999.0 * i / (n - 1))) for i in range(n)]


def step_config(name: str, n: Optional[int] = None, ragged: bool = False) -> StepConfig:
    if name == "tiny_f32":
        return StepConfig(name, "f32", 2, 64, [128, 128], 128, 128, [500, 999], 1.0,
                          SEED_BASE + 0, push_rows=128,
                          note="2 blocks x 2 frames x 8x8 tokens; t = {500 (head), 999}")
    if name == "cogvideo_bf16":
        return StepConfig(name, "bf16", 48, 64, [2700] * 4, 2700, 2700, _even_timesteps(4),
                          1.0 / 8.0, SEED_BASE + 1, push_rows=2700,
                          note="CogVideoX-like 480x720: 1350 tokens per latent frame")
    if name == "wan_bf16":
        return StepConfig(name, "bf16", 12, 128, [6240] * 8, 6240, 6240, _even_timesteps(8),
                          1.0, SEED_BASE + 2, push_rows=6240,
                          note="Wan-like 832x480: 1560 tokens per latent frame")
    if name == "longrun_steady_bf16":
        return StepConfig(name, "bf16", 24, 64, [2700] * 8, 2700, 2700, _even_timesteps(8),
                          1.0, SEED_BASE + 6, push_rows=2700,
                          note="steady state of the long run: 8 blocks of 2 latent frames x 1350 tokens")
    if name == "wan_paper_bf16":
        return StepConfig(name, "bf16", 12, 128, [12480] * 4, 12480, 12480, _even_timesteps(4),
                          1.0, SEED_BASE + 7, push_rows=12480,
                          note="blocks of 8 latent frames (the pages' block boundaries and 8-frame context)")
    if name == "sweep":
        if n is None:
            raise ValueError("sweep needs n (window tokens)")
        if n % 16:
            raise ValueError("sweep window must be a multiple of 16 tokens")
        frame = n // 16
        frames = [4, 4, 4, 3] if ragged else [4, 4, 4, 4]
        rows = [f * frame for f in frames]
        return StepConfig(f"sweep_{n}{'_ragged' if ragged else ''}", "bf16", 16, 128, rows,
                          n // 4, n // 4, [0] * 4, 1.0, SEED_BASE + 4 + (1 if ragged else 0),
                          push_rows=rows[0], random_timesteps=True,
                          note="4 blocks of 4 frames of n/16 tokens; ragged: last block 3 frames")
    raise KeyError(name)


def sweep_configs(ragged_too: bool = True) -> List[StepConfig]:
    out = []
    for n in [4096, 8192, 16384, 32768, 65536, 131072]:
        out.append(step_config("sweep", n))
        if ragged_too:
            out.append(step_config("sweep", n, ragged=True))
    return out


def run_config(name: str = "long_run") -> RunConfig:
    if name != "long_run":
        raise KeyError(name)
    return RunConfig(name, 24, 64, n_frames=257, frame_rows=1350, frames_per_block=2,
                     window_blocks=8, n_timesteps=50, seed=SEED_BASE + 3)

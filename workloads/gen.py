"""Seeded synthetic inputs (CPU ``torch.Generator``), shared by the oracle side and the GPU side.

Draw order for a window step is fixed: q, k, v, cache K, cache V, adaLN table, noise block,
then (sweep only) the per-block timesteps.  Every draw is float32 N(0,1) scaled by the
config's std, then rounded once to the config dtype (round-to-nearest-even for bf16).
The adaLN table stands in for the timestep MLP of a trained DiT: row t holds
(shift, scale, gate) vectors, each tanh(N(0,1)).
"""
from __future__ import annotations

from typing import Dict, List

import torch

from .configs import RunConfig, StepConfig


def to_dtype(x: torch.Tensor, dtype: str) -> torch.Tensor:
    if dtype == "f32":
        return x.to(torch.float32).contiguous()
    if dtype == "bf16":
        return x.to(torch.bfloat16).contiguous()
    raise ValueError(dtype)


def as_features(x: torch.Tensor, dtype: str) -> torch.Tensor:
    """Cached K/V enter the window step as stored features: f16 on the bf16 path (every bf16
    value in f16's normal range converts exactly), fp32 on the fp32 path."""
    return x.to(torch.float16).contiguous() if dtype == "bf16" else x.to(torch.float32).contiguous()


def _randn(g: torch.Generator, shape, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x


def make_step_inputs(cfg: StepConfig) -> Dict[str, object]:
    """Return CPU tensors for one window step of ``cfg``.

    Keys: q, k, v [n_win, hidden]; cache_k, cache_v [cache_capacity, hidden] (the first
    cache_len rows valid); table [table_rows, 3, hidden] fp32; noise [push_rows, hidden];
    timesteps (list[int], head first); row_offset (list[int], n_blocks + 1).
    """
    g = torch.Generator().manual_seed(cfg.seed)
    D = cfg.hidden
    out: Dict[str, object] = {}
    for key, rows in (("q", cfg.n_win), ("k", cfg.n_win), ("v", cfg.n_win),
                      ("cache_k", cfg.cache_capacity), ("cache_v", cfg.cache_capacity)):
        out[key] = to_dtype(_randn(g, (rows, D), cfg.qkv_std), cfg.dtype)
    out["table"] = torch.tanh(_randn(g, (cfg.table_rows, 3, D))).contiguous()
    out["noise"] = to_dtype(_randn(g, (cfg.push_rows, D)), cfg.dtype)
    if cfg.random_timesteps:
        t = torch.randint(0, cfg.table_rows, (cfg.n_blocks,), generator=g)
        out["timesteps"] = [int(x) for x in t.tolist()]
    else:
        out["timesteps"] = list(cfg.timesteps)
    out["row_offset"] = cfg.row_offset
    return out


def make_run_table(cfg: RunConfig) -> torch.Tensor:
    """adaLN table of the long run (first draw of the run's generator)."""
    g = torch.Generator().manual_seed(cfg.seed)
    return torch.tanh(_randn(g, (cfg.table_rows, 3, cfg.hidden))).contiguous()


def make_run_noise(cfg: RunConfig, dtype: str = "bf16") -> List[torch.Tensor]:
    """Noise blocks of the long run, in entry order, drawn after the table."""
    g = torch.Generator().manual_seed(cfg.seed)
    _randn(g, (cfg.table_rows, 3, cfg.hidden))  # advance past the table draw
    return [to_dtype(_randn(g, (rows, cfg.hidden)), dtype) for rows in cfg.block_rows]


def make_sublayer_weights(hidden: int, seed: int) -> Dict[str, torch.Tensor]:
    """Seeded stand-in weights of the DiT attention sublayer (trained weights are out of
    reach): W_qkv [3 hidden][hidden] and W_o [hidden][hidden] (out-features x in-features)
    drawn N(0, 1/hidden) so unit-variance inputs give unit-variance outputs, rounded once
    to bf16; biases N(0, 0.02^2) in float32.  Draw order: W_qkv, b_qkv, W_o, b_o."""
    g = torch.Generator().manual_seed(seed)
    s = 1.0 / float(hidden) ** 0.5
    w_qkv = _randn(g, (3 * hidden, hidden), s).to(torch.bfloat16).contiguous()
    b_qkv = _randn(g, (3 * hidden,), 0.02).contiguous()
    w_o = _randn(g, (hidden, hidden), s).to(torch.bfloat16).contiguous()
    b_o = _randn(g, (hidden,), 0.02).contiguous()
    return {"w_qkv": w_qkv, "b_qkv": b_qkv, "w_o": w_o, "b_o": b_o}


def make_noise_permutations(n_blocks: int, pool_frames: int, seed: int) -> List[List[int]]:
    """One seeded random permutation of the noise pool's frames per block (the random draw of
    the coordinated noise initialisation, an input to both sides)."""
    g = torch.Generator().manual_seed(seed)
    return [torch.randperm(pool_frames, generator=g).tolist() for _ in range(n_blocks)]


def make_run_pool(cfg: RunConfig, dtype: str = "bf16") -> torch.Tensor:
    """The noise pool of the long run with coordinated initialisation: the first window's
    noise, [window_blocks * frames_per_block, frame_rows, hidden], drawn after the table."""
    g = torch.Generator().manual_seed(cfg.seed + 1000)
    n = cfg.window_blocks * cfg.frames_per_block
    return to_dtype(_randn(g, (n, cfg.frame_rows, cfg.hidden)), dtype)

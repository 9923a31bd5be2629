"""The shape sweep (16x128 heads, bf16, window 4096..131072 tokens in 4 blocks, cache =
window/4, random per-block timesteps, a ragged last block variant) through the window step:
element-by-element against the oracle at the smallest size, sampled rows at every larger
power of two up to the maximum size, each size both regular and ragged (12 cases)."""
import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import assert_close, bytes_equal, sample_rows
from workloads import as_features, make_step_inputs, step_config

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _run(dp, cfg):
    x = make_step_inputs(cfg)
    H, hd, D, n = cfg.n_heads, cfg.head_dim, cfg.hidden, cfg.n_win
    blk = dp.blocks_from_table(x["table"].cuda(), x["timesteps"], cfg.block_rows)
    x["cache_k"], x["cache_v"] = as_features(x["cache_k"], cfg.dtype), as_features(x["cache_v"], cfg.dtype)
    cache = dp.KVCache(cfg.cache_capacity, D, torch.float16, k=x["cache_k"].cuda().view(1, -1, D),
                       v=x["cache_v"].cuda().view(1, -1, D), length=cfg.cache_len)
    kv = torch.empty(2, n, D, dtype=torch.float16, device="cuda")
    out = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
    dp.window_step(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), blk, cache, kv, out, H, hd, pop=True)
    dp.device_status()
    n0 = cfg.block_rows[0]
    assert cache.length == n0 and bytes_equal(cache.k[0, :n0], kv[0, :n0]) and bytes_equal(cache.v[0, :n0], kv[1, :n0])
    return x, out


@pytest.mark.parametrize("ragged", [False, True])
def test_sweep_4096_full(dp, ragged):
    cfg = step_config("sweep", 4096, ragged=ragged)
    x, out = _run(dp, cfg)
    mod = O.lookup(x["table"], x["timesteps"])
    want, _, _ = O.window_step(x["q"], x["k"], x["v"], x["cache_k"], x["cache_v"], cfg.cache_len, cfg.row_offset,
                               mod, cfg.n_heads, cfg.head_dim)
    assert_close(out.cpu().double().numpy(), want, "bf16", cfg.name)


@pytest.mark.parametrize("n", [8192, 16384, 32768, 65536, 131072])
@pytest.mark.parametrize("ragged", [False, True], ids=["regular", "ragged"])
def test_sweep_sampled(dp, n, ragged):
    cfg = step_config("sweep", n, ragged=ragged)
    x, out = _run(dp, cfg)
    rows = sample_rows(cfg.row_offset, n_extra=16, seed=n)
    got = out[rows].cpu().double().numpy()
    del out
    mod = O.lookup(x["table"], x["timesteps"])
    want, _, _ = O.window_step(x["q"], x["k"], x["v"], x["cache_k"], x["cache_v"], cfg.cache_len, cfg.row_offset,
                               mod, cfg.n_heads, cfg.head_dim, rows=rows)
    assert_close(got, want, "bf16", cfg.name)

"""Seeded synthetic inputs: determinism, shapes, dtypes and distributions."""
import numpy as np
import torch

from workloads import make_step_inputs, step_config, sweep_configs, run_config, make_run_noise


def test_step_inputs_deterministic_and_shaped():
    cfg = step_config("tiny_f32")
    a = make_step_inputs(cfg)
    b = make_step_inputs(cfg)
    for key in ("q", "k", "v", "cache_k", "cache_v", "table", "noise"):
        assert torch.equal(a[key], b[key])
    assert a["q"].shape == (256, 128) and a["q"].dtype == torch.float32
    assert a["cache_k"].shape == (128, 128)
    assert a["table"].shape == (1000, 3, 128)
    assert a["timesteps"] == [500, 999] and a["row_offset"] == [0, 128, 256]
    assert float(a["table"].abs().max()) < 1.0


def test_draw_order_q_first():
    cfg = step_config("tiny_f32")
    g = torch.Generator().manual_seed(cfg.seed)
    q = torch.randn(256, 128, generator=g, dtype=torch.float32)
    assert torch.equal(make_step_inputs(cfg)["q"], q)


def test_config_timesteps_and_sizes():
    c1 = step_config("cogvideo_bf16")
    assert c1.timesteps == [0, 333, 666, 999] and c1.n_win == 10800 and c1.hidden == 3072
    c2 = step_config("wan_bf16")
    assert c2.timesteps == [0, 143, 285, 428, 571, 714, 856, 999]
    assert c2.n_win == 49920 and c2.cache_len == 6240 and c2.hidden == 1536
    assert c1.attn_flop() == 4 * 10800 * 13500 * 64 * 48
    c3 = step_config("longrun_steady_bf16")
    rc = run_config()
    assert c3.block_rows == [rc.slot_rows] * rc.window_blocks and c3.cache_len == rc.slot_rows
    assert (c3.n_heads, c3.head_dim) == (rc.n_heads, rc.head_dim) and c3.n_win == 21600
    c4 = step_config("wan_paper_bf16")
    assert c4.block_rows == [8 * 1560] * 4 and c4.cache_len == 8 * 1560 and c4.hidden == 1536
    sw = sweep_configs()
    assert [c.n_win for c in sw[:2]] == [4096, 3840]
    assert sw[-1].cache_len == 131072 // 4 and sw[-1].block_rows == [32768, 32768, 32768, 24576]


def test_bf16_inputs_are_rounded_normals():
    cfg = step_config("cogvideo_bf16")
    cfg.block_rows = [64, 64]          # small slice of the same recipe
    cfg.cache_capacity = cfg.cache_len = 32
    cfg.push_rows = 64
    x = make_step_inputs(cfg)
    assert x["q"].dtype == torch.bfloat16
    s = float(x["q"].float().std())
    assert abs(s - 1.0 / 8.0) < 0.01
    t = make_step_inputs(step_config("sweep", 4096))["timesteps"]
    assert len(t) == 4 and all(0 <= v < 1000 for v in t)


def test_run_noise_blocks():
    rc = run_config()
    rc.n_frames, rc.frame_rows = 5, 3        # tiny slice of the run recipe
    blocks = make_run_noise(rc)
    assert [b.shape[0] for b in blocks] == [6, 6, 3]
    assert all(b.dtype == torch.bfloat16 for b in blocks)

"""Host-side logic of bench.py (no GPU): which measured peak a roofline uses, the algorithmic
bytes of the HBM-bound stages, and the reference arm's JSON line (the CPU oracle timed on a
bounded sample of a small workload)."""
import argparse

import pytest

import bench
from workloads import step_config

PEAKS = {"hbm_gbs": 6552.6, "bf16_tflops": 1667.9, "bf16_tflops_sustained": 1387.6, "source": "measured"}


def test_peak_follows_the_clock_record():
    # power cap over a long timed region: the sustained GEMM peak (measured the same way)
    pk = bench.choose_peak(PEAKS, {"reasons": ["sw_power_cap"]}, 5.0)
    assert pk["peak"] == 1387.6 and pk["kind"].startswith("bf16_tflops_sustained")
    # no cap, or a cap over a region shorter than a second: the burst peak
    assert bench.choose_peak(PEAKS, {"reasons": []}, 5.0)["peak"] == 1667.9
    assert bench.choose_peak(PEAKS, {"reasons": ["sw_power_cap"]}, 0.4)["peak"] == 1667.9
    assert bench.choose_peak(PEAKS, None, 5.0)["peak"] == 1667.9
    f = bench.roofline_fracs(1000.0, pk)
    assert f["frac"] == pytest.approx(1000 / 1387.6)
    assert f["frac_of_burst"] == pytest.approx(1000 / 1667.9)
    assert f["frac_of_sustained"] == pytest.approx(1000 / 1387.6)
    assert bench.roofline_fracs(None, pk)["frac"] is None


def test_hbm_stage_bytes_are_the_algorithmic_ones():
    cfg = step_config("cogvideo_bf16")
    D, eb = cfg.hidden, 2
    r = {"mod_ms": 0.05, "adv_ms": 0.02, "mod_alone_ms": 0.04, "adv_alone_ms": 0.01}
    out = bench.stage_hbm(cfg, r, PEAKS)
    assert out["modulate"]["bytes"] == 4 * cfg.n_win * D * eb
    # the advance: the head block's k', v' read and written (4 n_exit rows), the noise block read
    # and written once (2 n_push rows); the mirror half of the latent ring is reported apart
    assert out["advance"]["bytes"] == (4 * cfg.block_rows[0] + 2 * cfg.push_rows) * D * eb
    assert out["advance"]["mirror_write_bytes"] == cfg.push_rows * D * eb
    assert out["advance"]["achieved_gbs"] == pytest.approx(out["advance"]["bytes"] / 0.02e-3 / 1e9)
    assert out["modulate_alone"]["bytes"] == out["modulate"]["bytes"]
    assert out["advance_cache_alone"]["bytes"] == 4 * cfg.block_rows[0] * D * eb
    assert out["modulate_alone"]["frac"] == pytest.approx(out["modulate"]["bytes"] / 0.04e-3 / 1e9 / 6552.6)


def test_reference_arm_line():
    args = argparse.Namespace(config="tiny_f32", steps=3, warmup=3, gpus=1)
    line = bench.reference_arm(args)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "tokens/s"
    assert line["higher_is_better"] is True and line["vs_baseline"] is None and line["steps"] == 3
    cfg = step_config("tiny_f32")
    assert line["value"] == pytest.approx(cfg.n_win / (line["ms_per_step"] / 1e3))
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"].startswith("tiny_f32")


def test_default_workload_is_the_largest_single_gpu_window():
    cfg = bench.workload(bench.DEFAULT_CONFIG)
    assert cfg.n_win == 131072 and cfg.cache_len == 32768 and (cfg.n_heads, cfg.head_dim) == (16, 128)
    assert set(bench.EXTRA_CONFIGS) == {"wan_bf16", "longrun_steady_bf16", "long_run"}

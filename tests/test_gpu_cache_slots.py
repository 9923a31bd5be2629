"""Attention over several cache slots (DP_STEP_CACHE_ALL_SLOTS: the K/V of the last n_slots
exited blocks, the pages' NumC frames of context) against the oracle, through the C ABI:
a preset ring with full, ragged and empty slots (tensor cores at both head dims, and the
fp32 path), and the long run with four blocks of context."""
import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import assert_close, sample_rows
from workloads import make_run_noise, make_run_table, run_config

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("dtype,H,hd,cap,rows", [("bf16", 4, 64, 300, [300, 211]), ("bf16", 2, 128, 300, [256, 129]),
                                                 ("f32", 2, 64, 128, [128, 77])])
def test_window_step_reads_every_cache_slot(dp, dtype, H, hd, cap, rows):
    D = H * hd
    n = sum(rows)
    g = torch.Generator().manual_seed(11)
    wdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    fdt = torch.float16 if dtype == "bf16" else torch.float32
    q, k, v = (torch.randn(n, D, generator=g).to(wdt) for _ in range(3))
    ring_k = torch.randn(3, cap, D, generator=g).to(fdt)
    ring_v = torch.randn(3, cap, D, generator=g).to(fdt)
    lens = [cap, 123, 0]                       # full, ragged, empty
    table = torch.tanh(torch.randn(1000, 3, D, generator=g))
    ts = [100, 900]
    blk = dp.blocks_from_table(table.cuda(), ts, rows)
    mod = O.lookup(table, ts)
    ro = [0, rows[0], n]
    kv = torch.empty(2, n, D, dtype=fdt, device="cuda")
    out = torch.empty(n, D, dtype=wdt, device="cuda")
    tdt = "bf16" if dtype == "bf16" else "f32"
    for all_slots in (True, False):
        cache = dp.KVCache(cap, D, fdt, n_slots=3, k=ring_k.cuda().clone(), v=ring_v.cuda().clone())
        for s, L in enumerate(lens):
            cache.desc.len[s] = L
        cache.desc.n_advances = 5                  # most recently written slot: (5 - 1) % 3 = 1
        dp.window_step(q.cuda(), k.cuda(), v.cuda(), blk, cache, kv, out, H, hd, cache_all_slots=all_slots)
        dp.device_status()
        if all_slots:
            ck = torch.cat([ring_k[0, :cap], ring_k[1, :123]])
            cv = torch.cat([ring_v[0, :cap], ring_v[1, :123]])
        else:
            ck, cv = ring_k[1, :123], ring_v[1, :123]
        # the oracle modulates the raw window k, v itself, in float64
        want, _, _ = O.window_step(q, k, v, ck, cv, ck.shape[0], ro, mod, H, hd)
        assert_close(out.cpu().double().numpy(), want, tdt, f"all_slots={all_slots}")


def test_long_run_with_four_blocks_of_context(dp):
    """The long run (2-frame blocks, window of 8) with a 4-slot cache read whole: 8 latent
    frames of context, the pages' NumC = 8, through its first 121 steps (the first exit comes
    after step 49; the context is full from the fourth exit on)."""
    rc = run_config()
    H, hd, D, W, T = rc.n_heads, rc.head_dim, rc.hidden, rc.window_blocks, rc.n_timesteps
    noise_cpu = make_run_noise(rc)
    table_cpu = make_run_table(rc)
    noise = [b.cuda() for b in noise_cpu]
    table = table_cpu.cuda()
    tau = O.timestep_schedule(T)
    run = O.LongRun(noise_cpu, table_cpu, H, hd, W, T, context_blocks=4)
    cache = dp.KVCache(rc.slot_rows, D, torch.float16, n_slots=4)
    queue = dp.Queue(W, rc.slot_rows, D)
    n_max = W * rc.slot_rows
    kv = torch.empty(2 * n_max * D, dtype=torch.float16, device="cuda")
    out = torch.empty(n_max, D, dtype=torch.bfloat16, device="cuda")
    check = {50, 57, 69, 120}
    results = {}

    def on_step(step, n, popped, pushed):
        if step in check:
            ro = [0]
            for b in run.schedule[step]["live"]:
                ro.append(ro[-1] + noise_cpu[b].shape[0])
            rows = sample_rows(ro, n_extra=16, seed=step)
            results[step] = (out[rows].cpu().double().numpy(), rows)

    steps = dp.run_fifo(noise, table, tau, W, cache, queue, kv, out, H, hd, on_step=on_step, max_steps=121,
                        cache_all_slots=True)
    dp.device_status()
    assert steps == 121
    assert cache.n_advances == sum(1 for u in range(121) if run.schedule[u]["pop_after"])
    for step, (got, rows) in sorted(results.items()):
        want, ro, t, L = run.step(step, rows=rows)
        assert L == min(4, sum(1 for u in range(step) if run.schedule[u]["pop_after"])) * rc.slot_rows
        assert_close(got, want, "bf16", f"context of 4 blocks, step {step}")

"""Coordinated noise initialisation on the GPU, through the C ABI: the frame-gather push is
bit-exact against the pool's frames, and the long run with coordinated pushes matches the
oracle (the host-side selection rule is checked against the oracle's in
tests/test_noise_init_host.py)."""
import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import assert_close, bytes_equal, sample_rows
from workloads import make_noise_permutations, make_run_pool, make_run_table, run_config

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_queue_push_frames_gathers_pool_frames(dp):
    D, fr = 256, 100
    g = torch.Generator().manual_seed(1)
    pool = torch.randn(6, fr, D, generator=g).to(torch.bfloat16).cuda()
    q = dp.Queue(3, 3 * fr, D)
    dp.queue_push_frames(q, pool, [4, 1, 5])
    dp.queue_push_frames(q, pool, [0, 2, 3])
    dp.queue_push_frames(q, pool, [5, 4])          # a short final block (2 frames)
    torch.cuda.synchronize()
    want = torch.cat([pool[4], pool[1], pool[5], pool[0], pool[2], pool[3], pool[5], pool[4]])
    assert bytes_equal(q.window(), want)
    assert [q.desc.rows[i] for i in range(3)] == [300, 300, 200]
    with pytest.raises(dp.DpError):
        dp.queue_push_frames(dp.Queue(2, 3 * fr, D), pool, [6])      # index outside the pool


def test_long_run_with_coordinated_noise(dp):
    rc = run_config()
    H, hd, D, W, T = rc.n_heads, rc.head_dim, rc.hidden, rc.window_blocks, rc.n_timesteps
    pool_cpu = make_run_pool(rc)                                  # [16, 1350, D] bf16
    frames = [r // rc.frame_rows for r in rc.block_rows]          # 2 ... 2, 1
    perms = make_noise_permutations(len(frames), pool_cpu.shape[0], seed=rc.seed + 2000)
    lists = dp.coordinated_schedule(frames, W, perms)
    sched = O.coordinated_schedule(frames, W, perms)
    assert lists == sched
    latents = [O.gather_frames(pool_cpu, f) for f in sched]
    run = O.LongRun(latents, make_run_table(rc), H, hd, W, T)
    table = make_run_table(rc).cuda()
    tau = O.timestep_schedule(T)
    cache = dp.KVCache(rc.slot_rows, D, torch.float16)
    queue = dp.Queue(W, rc.slot_rows, D)
    n_max = W * rc.slot_rows
    kv = torch.empty(2 * n_max * D, dtype=torch.float16, device="cuda")
    out = torch.empty(n_max, D, dtype=torch.bfloat16, device="cuda")
    pool = pool_cpu.cuda()
    check = {30, 60, 120}
    results = {}

    def on_step(step, n, popped, pushed):
        if step in check:
            torch.cuda.synchronize()
            live = run.schedule[step + 1]["live"]
            win = torch.from_numpy(np.concatenate([latents[b] for b in live])).to(torch.bfloat16)
            assert bytes_equal(queue.window().cpu(), win), step         # queue after the step's push
            ro = [0]
            for b in run.schedule[step]["live"]:
                ro.append(ro[-1] + latents[b].shape[0])
            rows = sample_rows(ro, n_extra=16, seed=step)
            results[step] = (out[rows].cpu().double().numpy(), rows)

    steps = dp.run_fifo(lists, table, tau, W, cache, queue, kv, out, H, hd, on_step=on_step, max_steps=121,
                        frame_pool=(pool, lists))
    dp.device_status()
    assert steps == 121
    for step, (got, rows) in sorted(results.items()):
        want, ro, t, L = run.step(step, rows=rows)
        assert_close(got, want, "bf16", f"coordinated noise, step {step}")

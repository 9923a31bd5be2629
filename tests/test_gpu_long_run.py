"""The full long-video queue run (257 latent frames of 30x45 tokens in 2-frame blocks, a
window of 8 blocks, 50 staggered timesteps per block, 24x64 heads, bf16): every step runs
through the CUDA path; outputs are compared with the oracle at sampled steps, and the queue
and cache contents are checked at every advance."""
import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import assert_close, bytes_equal, sample_rows
from workloads import make_run_noise, make_run_table, run_config

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

# warm-up shapes (1..8 blocks), right after the first advances, steady state, the last step
CHECK_STEPS = {0, 6, 12, 18, 25, 31, 37, 43, 50, 56, 400, 849}


def test_long_run_matches_oracle(dp):
    rc = run_config()
    H, hd, D, W, T = rc.n_heads, rc.head_dim, rc.hidden, rc.window_blocks, rc.n_timesteps
    noise_cpu = make_run_noise(rc)
    table_cpu = make_run_table(rc)
    noise = [b.cuda() for b in noise_cpu]
    table = table_cpu.cuda()
    tau = O.timestep_schedule(T)
    run = O.LongRun(noise_cpu, table_cpu, H, hd, W, T)
    total = len(run.schedule)
    cache = dp.KVCache(rc.slot_rows, D, torch.float16)
    queue = dp.Queue(W, rc.slot_rows, D)
    n_max = W * rc.slot_rows
    kv = torch.empty(2 * n_max * D, dtype=torch.float16, device="cuda")  # k' then v' at n_win * D
    out = torch.empty(n_max, D, dtype=torch.bfloat16, device="cuda")
    m_last = O.lookup(table_cpu, [tau[T - 1]])
    live = [0]
    advances = []
    results = {}

    def on_step(step, n, popped, pushed):
        sched = run.schedule[step]
        kp, vp = kv[:n * D].view(n, D), kv[n * D:2 * n * D].view(n, D)
        assert live == sched["live"], (step, live, sched["live"])
        assert n == sum(noise_cpu[b].shape[0] for b in live)
        if step in CHECK_STEPS:
            ro = [0]
            for b in live:
                ro.append(ro[-1] + noise_cpu[b].shape[0])
            rows = sample_rows(ro, n_extra=24, seed=step)
            results[step] = (out[rows].cpu().double().numpy(), rows)
        if popped:
            b = live.pop(0)
            assert sched["pop_after"] == [b]
            n_exit = noise_cpu[b].shape[0]
            torch.cuda.synchronize()
            # the cache is the exited block's k'/v' from this (its last) evaluation
            assert cache.length == n_exit
            assert bytes_equal(cache.k[0, :n_exit], kp[:n_exit])
            assert bytes_equal(cache.v[0, :n_exit], vp[:n_exit])
            if len(advances) % 16 == 0 or b == len(noise_cpu) - 1:
                want = O.modulate_rounded(noise_cpu[b], [0, n_exit], m_last, "f16")
                assert np.array_equal(cache.k[0, :n_exit].cpu().double().numpy(), want)
            advances.append(b)
        else:
            assert sched["pop_after"] == []
        if pushed is not None:
            assert sched["push_after"] == [pushed]
            live.append(pushed)
        else:
            assert sched["push_after"] == []
        # after the step the queue holds exactly the next step's live blocks, head first
        if live and (step % 25 == 0 or popped):
            assert step + 1 < total and live == run.schedule[step + 1]["live"]
            torch.cuda.synchronize()
            assert bytes_equal(queue.window(), torch.cat([noise[b] for b in live]))

    steps = dp.run_fifo(noise, table, tau, W, cache, queue, kv, out, H, hd, on_step=on_step)
    dp.device_status()
    assert steps == total == 850
    assert advances == list(range(len(noise_cpu)))
    assert queue.count == 0 and queue.desc.n_pushed == 129 and queue.desc.n_popped == 129
    assert cache.n_advances == 129
    for step, (got, rows) in sorted(results.items()):
        want, ro, t, L = run.step(step, rows=rows)
        assert_close(got, want, "bf16", f"long run step {step}")


def test_long_run_checkpoint_and_resume_is_bit_identical(dp):
    """The run stopped at a steady-state step, checkpointed to host memory through
    torch.save, restored into new buffers and continued gives, at every later step, the
    outputs of the uninterrupted run bit for bit, and the same final cache and queue."""
    import io
    rc = run_config()
    H, hd, D, W, T = rc.n_heads, rc.head_dim, rc.hidden, rc.window_blocks, rc.n_timesteps
    noise = [b.cuda() for b in make_run_noise(rc)]
    table = make_run_table(rc).cuda()
    tau = O.timestep_schedule(T)
    n_max = W * rc.slot_rows
    kv = torch.empty(2 * n_max * D, dtype=torch.float16, device="cuda")
    out = torch.empty(n_max, D, dtype=torch.bfloat16, device="cuda")

    def sums_into(lst):
        return lambda step, n, popped, pushed: lst.append(out[:n].view(torch.int16).sum(dtype=torch.int64))

    ref = []
    cache, queue = dp.KVCache(rc.slot_rows, D, torch.float16), dp.Queue(W, rc.slot_rows, D)
    assert dp.run_fifo(noise, table, tau, W, cache, queue, kv, out, H, hd, on_step=sums_into(ref)) == 850
    got = []
    cache2, queue2 = dp.KVCache(rc.slot_rows, D, torch.float16), dp.Queue(W, rc.slot_rows, D)
    state = dp.FifoState()
    assert dp.run_fifo(noise, table, tau, W, cache2, queue2, kv, out, H, hd, on_step=sums_into(got),
                       max_steps=300, state=state) == 300
    buf = io.BytesIO()
    torch.save(dp.checkpoint(queue2, cache2, state), buf)
    del queue2, cache2
    kv.fill_(0)
    buf.seek(0)
    queue3, cache3, state3 = dp.restore(torch.load(buf))
    assert state3.step == 300
    assert dp.run_fifo(noise, table, tau, W, cache3, queue3, kv, out, H, hd, on_step=sums_into(got),
                       state=state3) == 850
    dp.device_status()
    assert torch.equal(torch.stack(got).cpu(), torch.stack(ref).cpu())
    assert cache3.desc.n_advances == cache.desc.n_advances == len(noise) and cache3.length == cache.length
    assert bytes_equal(cache3.k, cache.k) and bytes_equal(cache3.v, cache.v)
    assert queue3.count == queue.count == 0 and queue3.desc.n_popped == queue.desc.n_popped


def test_long_run_alternating_output_buffers(dp):
    """run_fifo with a list of output buffers writes step s into buffer s % 2, with the same
    values as a run with one buffer."""
    rc = run_config()
    H, hd, D, W, T = rc.n_heads, rc.head_dim, rc.hidden, rc.window_blocks, rc.n_timesteps
    noise = [b.cuda() for b in make_run_noise(rc)]
    table = make_run_table(rc).cuda()
    tau = O.timestep_schedule(T)
    n_max = W * rc.slot_rows
    kv = torch.empty(2 * n_max * D, dtype=torch.float16, device="cuda")
    one = torch.empty(n_max, D, dtype=torch.bfloat16, device="cuda")
    two = [torch.empty_like(one), torch.empty_like(one)]
    a, b = [], []

    def grab(lst, buf_of):
        return lambda step, n, popped, pushed: lst.append(buf_of(step)[:n].clone())

    dp.run_fifo(noise, table, tau, W, dp.KVCache(rc.slot_rows, D, torch.float16), dp.Queue(W, rc.slot_rows, D), kv,
                one, H, hd, on_step=grab(a, lambda s: one), max_steps=60)
    dp.run_fifo(noise, table, tau, W, dp.KVCache(rc.slot_rows, D, torch.float16), dp.Queue(W, rc.slot_rows, D), kv,
                two, H, hd, on_step=grab(b, lambda s: two[s % 2]), max_steps=60)
    dp.device_status()
    assert len(a) == len(b) == 60
    assert all(bytes_equal(x, y) for x, y in zip(a, b))

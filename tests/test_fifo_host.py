"""The queue's schedule and the coordinated noise selection behind the C ABI (no GPU: these
calls read and write host descriptors only) against the oracle: dp_fifo_plan / dp_fifo_commit
reproduce oracle.long_run_schedule step for step (the long run's 850 steps, and random
video lengths, windows and timestep counts), and dp_coordinated_frames reproduces
oracle.coordinated_schedule block for block."""
import ctypes

import pytest
from hypothesis import given, settings, strategies as st

import long_video_diffusion_b200 as dp
import oracle as O
from workloads import make_noise_permutations, run_config

FAKE = 0x7f0000000000
HIDDEN = 128


def _queue(n_slots, slot_rows=64):
    q = dp.DpQueue()
    q.latent = FAKE
    q.slot_rows, q.hidden, q.n_slots, q.head, q.count, q.dtype = slot_rows, HIDDEN, n_slots, 0, 0, dp.BF16
    return q


def _model_push(q, rows):
    """What a push does to the host descriptor (dp_queue_push without its copy)."""
    q.rows[q.count], q.evals[q.count] = rows, 0
    q.count += 1
    q.n_pushed += 1


def _model_step(q, pop):
    """What a window step does to the descriptor: every live block is evaluated once; a pop
    removes the head."""
    for i in range(q.count):
        q.evals[i] += 1
    if pop:
        assert dp._lib.dp_queue_pop(ctypes.byref(q)) == dp.OK


def _walk(n_blocks, T, W, rows_of, extra_slots=0):
    """Drive the schedule through a model queue; return the per-step records."""
    f = dp.DpFifo()
    assert dp._lib.dp_fifo_init(ctypes.byref(f), n_blocks, T, W) == dp.OK
    q = _queue(W + extra_slots)
    plan = dp.DpFifoStep()
    steps = []
    for _ in range(100000):
        assert dp._lib.dp_fifo_plan(ctypes.byref(f), ctypes.byref(q), ctypes.byref(plan)) == dp.OK
        if plan.done:
            break
        if plan.push_before >= 0:
            assert plan.push_before == 0 and f.step == 0
            _model_push(q, rows_of(0))
            assert dp._lib.dp_fifo_commit(ctypes.byref(f), ctypes.byref(plan)) == dp.OK
            continue
        live_count = q.count
        steps.append({"step": f.step, "count": live_count, "pop": bool(plan.pop), "exit_rows": plan.exit_rows,
                      "push": plan.push_after, "head_evals": q.evals[0], "ctx": (plan.ctx_rows or 0, plan.ctx_n),
                      "head": q.head})
        _model_step(q, plan.pop)
        if plan.push_after >= 0:
            _model_push(q, rows_of(plan.push_after))
        assert dp._lib.dp_fifo_commit(ctypes.byref(f), ctypes.byref(plan)) == dp.OK
    else:
        raise AssertionError("schedule did not finish")
    assert q.count == 0 and f.next_block == n_blocks
    return steps


def _check_against_oracle(n_blocks, T, W, rows_of):
    sched = O.long_run_schedule(n_blocks, W, T)
    got = _walk(n_blocks, T, W, rows_of)
    assert len(got) == len(sched)
    for g, s in zip(got, sched):
        assert g["step"] == s["step"]
        assert g["count"] == len(s["live"])
        assert g["head_evals"] == s["k"][0]
        assert g["pop"] == bool(s["pop_after"])
        assert g["exit_rows"] == (rows_of(s["pop_after"][0]) if s["pop_after"] else 0)
        assert g["push"] == (s["push_after"][0] if s["push_after"] else -1)
    return got


def test_long_run_schedule_matches_the_oracle_at_every_step():
    rc = run_config()
    rows = rc.block_rows
    got = _check_against_oracle(len(rows), rc.n_timesteps, rc.window_blocks, lambda b: rows[b])
    assert len(got) == 850
    assert sum(g["pop"] for g in got) == 129
    assert sum(g["push"] >= 0 for g in got) == 128          # block 0 enters before the first step
    for b in range(len(rows)):
        assert dp.fifo_entry_step(b, rc.n_timesteps, rc.window_blocks) == O.entry_step(b, rc.n_timesteps,
                                                                                       rc.window_blocks)


@settings(max_examples=150, deadline=None)
@given(st.integers(1, 40), st.integers(1, dp.MAX_SLOTS), st.integers(0, 30), st.integers(1, 64))
def test_random_schedules_match_the_oracle(n_blocks, W, dT, last_rows):
    T = W + dT
    _check_against_oracle(n_blocks, T, W, lambda b: 64 if b < n_blocks - 1 else last_rows)


def test_context_rows_behind_the_head():
    """With one slot more than the window, the plan points at the latent slot behind the head
    (the block that left last) from the step after the first exit on; with no spare slot it
    points nowhere."""
    W, T = 4, 8
    got = _walk(10, T, W, lambda b: 64, extra_slots=1)
    first_pop = next(i for i, g in enumerate(got) if g["pop"])
    for i, g in enumerate(got):
        if i <= first_pop:
            assert g["ctx"] == (0, 0)
        else:
            behind = (g["head"] + W) % (W + 1)
            assert g["ctx"] == (FAKE + behind * 64 * HIDDEN * 2, 64)
    for g in _walk(10, T, W, lambda b: 64):
        assert g["ctx"] == (0, 0)


def test_plan_rejects_a_queue_that_does_not_match():
    f = dp.DpFifo()
    assert dp._lib.dp_fifo_init(ctypes.byref(f), 5, 8, 4) == dp.OK
    q = _queue(4)
    plan = dp.DpFifoStep()
    _model_push(q, 64)
    _model_push(q, 64)                     # two blocks before the first step: not the schedule
    assert dp._lib.dp_fifo_plan(ctypes.byref(f), ctypes.byref(q), ctypes.byref(plan)) == dp.ERR_INVALID_ARG
    assert dp._lib.dp_fifo_init(ctypes.byref(f), 5, 3, 4) == dp.ERR_INVALID_ARG    # T < W
    assert dp._lib.dp_fifo_init(ctypes.byref(f), 0, 8, 4) == dp.ERR_INVALID_ARG
    out = ctypes.c_int64()
    assert dp._lib.dp_fifo_entry_step(3, 2, 4, ctypes.byref(out)) == dp.ERR_INVALID_ARG


def test_commit_rejects_a_plan_that_skips_the_entering_block():
    f = dp.DpFifo()
    assert dp._lib.dp_fifo_init(ctypes.byref(f), 5, 4, 4) == dp.OK   # T = W: one block enters every step
    q = _queue(4)
    plan = dp.DpFifoStep()
    assert dp._lib.dp_fifo_plan(ctypes.byref(f), ctypes.byref(q), ctypes.byref(plan)) == dp.OK
    _model_push(q, 64)
    assert dp._lib.dp_fifo_commit(ctypes.byref(f), ctypes.byref(plan)) == dp.OK
    assert dp._lib.dp_fifo_plan(ctypes.byref(f), ctypes.byref(q), ctypes.byref(plan)) == dp.OK
    assert plan.push_after == 1
    plan.push_after = -1
    assert dp._lib.dp_fifo_commit(ctypes.byref(f), ctypes.byref(plan)) == dp.ERR_INVALID_ARG
    assert f.step == 0


@pytest.mark.parametrize("W,frames", [(8, [2] * 128 + [1]), (4, [3, 3, 2, 3, 3, 1]), (3, [1, 1, 1, 1, 1]),
                                      (2, [5])])
def test_coordinated_selection_matches_the_oracle(W, frames):
    pool = sum(frames[:W])
    perms = make_noise_permutations(len(frames), pool, seed=9 + W)
    want = O.coordinated_schedule(frames, W, perms)
    assert dp.coordinated_schedule(frames, W, perms) == want


def test_coordinated_selection_rejects_bad_input():
    frames = [2, 2, 2]
    with pytest.raises(dp.DpError):
        dp.coordinated_frames(frames, 2, 2, [0, 1], [0, 1, 1, 3])          # not a permutation
    with pytest.raises(dp.DpError):
        dp.coordinated_frames([2, 2, 4], 2, 2, [0, 1], [3, 2, 1, 0])        # 2 frames left, 4 needed
    with pytest.raises(dp.DpError):
        dp.coordinated_frames(frames, 2, 3, [], None)                        # no block 3
    assert dp.coordinated_frames(frames, 2, 2, [0, 1], [1, 3, 0, 2]) == [3, 2]
    assert dp.coordinated_frames(frames, 2, 1, [0, 1], None) == [2, 3]

"""Property tests of the library's host-side queue logic against a plain Python model (no GPU:
these calls only read and write the host descriptors; the table and latent pointers are
never dereferenced)."""
import ctypes

from hypothesis import given, settings, strategies as st

import long_video_diffusion_b200 as dp

FAKE = 0x7f0000000000
HIDDEN = 128


@st.composite
def queues(draw):
    n_slots = draw(st.integers(1, dp.MAX_SLOTS))
    slot_rows = draw(st.sampled_from([16, 64, 128]))
    count = draw(st.integers(0, n_slots))
    head = draw(st.integers(0, n_slots - 1))
    rows = [draw(st.integers(1, slot_rows)) for _ in range(count)]
    n_tau = draw(st.integers(1, 60))
    evals = [draw(st.integers(0, n_tau - 1)) for _ in range(count)]
    tau = [draw(st.integers(0, 999)) for _ in range(n_tau)]
    q = dp.DpQueue()
    q.latent = FAKE + (1 << 24)
    q.slot_rows, q.hidden, q.n_slots, q.head, q.count, q.dtype = slot_rows, HIDDEN, n_slots, head, count, dp.BF16
    q.n_pushed, q.n_popped = draw(st.integers(count, 500)), draw(st.integers(0, 500))
    for i in range(count):
        q.rows[i], q.evals[i] = rows[i], evals[i]
    return q, tau


@settings(max_examples=300, deadline=None)
@given(queues())
def test_queue_blocks_matches_model(qt):
    q, tau = qt
    out = dp.DpBlocks()
    win = ctypes.c_void_p()
    n = ctypes.c_int64()
    ta = (ctypes.c_int32 * len(tau))(*tau)
    st_ = dp._lib.dp_queue_blocks(ctypes.byref(q), ctypes.c_void_p(FAKE), 1000, ta, len(tau), ctypes.byref(out),
                                  ctypes.byref(win), ctypes.byref(n))
    if q.count == 0:
        assert st_ == dp.ERR_EMPTY
        return
    assert st_ == dp.OK
    rows = [q.rows[i] for i in range(q.count)]
    offs = [0]
    for r in rows:
        offs.append(offs[-1] + r)
    assert out.n_blocks == q.count and out.offsets == offs and n.value == offs[-1]
    for i in range(q.count):       # block i reads the table row of its own timestep
        assert out.mod[i] == FAKE + tau[q.evals[i]] * 3 * HIDDEN * 4
    assert win.value == q.latent + q.head * q.slot_rows * HIDDEN * 2   # the head slot of the mirrored ring


@settings(max_examples=300, deadline=None)
@given(queues(), st.integers(1, 20))
def test_pops_match_model(qt, n_pops):
    q, _ = qt
    model = {"head": q.head, "count": q.count, "popped": q.n_popped,
             "rows": [q.rows[i] for i in range(q.count)], "evals": [q.evals[i] for i in range(q.count)]}
    for _ in range(n_pops):
        st_ = dp._lib.dp_queue_pop(ctypes.byref(q))
        if model["count"] == 0:
            assert st_ == dp.ERR_EMPTY
            break
        assert st_ == dp.OK
        model["head"] = (model["head"] + 1) % q.n_slots
        model["count"] -= 1
        model["popped"] += 1
        model["rows"].pop(0)
        model["evals"].pop(0)
        assert (q.head, q.count, q.n_popped) == (model["head"], model["count"], model["popped"])
        assert [q.rows[i] for i in range(q.count)] == model["rows"]
        assert [q.evals[i] for i in range(q.count)] == model["evals"]


@settings(max_examples=200, deadline=None)
@given(queues())
def test_queue_blocks_rejects_finished_blocks(qt):
    q, tau = qt
    if q.count == 0:
        return
    q.evals[q.count - 1] = len(tau)      # one evaluation too many
    out = dp.DpBlocks()
    ta = (ctypes.c_int32 * len(tau))(*tau)
    assert dp._lib.dp_queue_blocks(ctypes.byref(q), ctypes.c_void_p(FAKE), 1000, ta, len(tau), ctypes.byref(out),
                                   ctypes.byref(ctypes.c_void_p()), ctypes.byref(ctypes.c_int64())) == dp.ERR_INVALID_ARG

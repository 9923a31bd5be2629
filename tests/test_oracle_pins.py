"""Pins for the CPU oracle: each check compares it with something other than itself
(brute-force loops, closed forms, a library routine, invariants), chosen so that a dropped
term, a wrong sign or index, or a transposed operand fails at least one of them."""
import math

import numpy as np
import pytest
import torch

import oracle as O


def _rng(seed=0):
    return np.random.default_rng(seed)


def _mod(rng, B, D, zero=False, gate_one=False):
    m = np.tanh(rng.standard_normal((B, 3, D)))
    if zero:
        m[:, 0] = 0.0
        m[:, 1] = 0.0
    if gate_one:
        m[:, 2] = 1.0
    return m


# --------------------------------------------------------------------------- modulation

def test_modulate_zero_shift_scale_is_identity_bitwise():
    rng = _rng(1)
    x = rng.standard_normal((37, 24))
    mod = _mod(rng, 3, 24, zero=True)
    y = O.modulate(x, [0, 5, 20, 37], mod)
    assert np.array_equal(y, x)


def test_modulate_scale_minus_one_returns_each_blocks_shift():
    # x * (1 + (-1)) + shift = shift: pins the row -> block map and the channel index
    rng = _rng(2)
    ro = [0, 3, 3, 10, 17]          # includes an empty block
    D = 16
    x = rng.standard_normal((17, D)) * 100.0
    mod = _mod(rng, 4, D)
    mod[:, 1, :] = -1.0
    y = O.modulate(x, ro, mod)
    for b in range(4):
        for i in range(ro[b], ro[b + 1]):
            assert np.array_equal(y[i], mod[b, 0])


def test_row_blocks_rejects_bad_offsets():
    with pytest.raises(ValueError):
        O.row_blocks([0, 5, 4], 4)
    with pytest.raises(ValueError):
        O.row_blocks([1, 4], 4)
    with pytest.raises(ValueError):
        O.row_blocks([0, 3], 4)


def test_modulate_rounded_hand_cases():
    # 1.0 * 1.5 + 0.25 = 1.75 exactly; 1 + 2^-9 rounds to 1.0 in bf16 (below half an ulp);
    # 1 + 3 * 2^-9 = 1 + 0.75 ulp rounds up to 1 + 2^-7.
    x = np.array([[1.0, 1.0, 1.0, -2.0]])
    mod = np.zeros((1, 3, 4))
    mod[0, 1] = [0.5, 2.0 ** -9, 3 * 2.0 ** -9, 0.0]
    mod[0, 0] = [0.25, 0.0, 0.0, 0.5]
    y = O.modulate_rounded(x, [0, 1], mod, "bf16")
    assert y.tolist() == [[1.75, 1.0, 1.0 + 2.0 ** -7, -1.5]]


def test_modulate_rounded_f16_hand_cases():
    # f16 has 10 fraction bits: 1 + 2^-11 is a tie and rounds to even (1.0); 1 + 3 * 2^-12
    # rounds up to 1 + 2^-10; 60000 * 2 saturates at 65504 instead of overflowing
    x = np.array([[1.0, 1.0, 60000.0, -60000.0]])
    mod = np.zeros((1, 3, 4))
    mod[0, 1] = [2.0 ** -11, 3 * 2.0 ** -12, 1.0, 1.0]
    y = O.modulate_rounded(x, [0, 1], mod, "f16")
    assert y.tolist() == [[1.0, 1.0 + 2.0 ** -10, 65504.0, -65504.0]]


def test_modulate_rounded_within_one_bf16_rounding():
    rng = _rng(3)
    x = torch.randn(64, 32, dtype=torch.float32).to(torch.bfloat16)
    mod = _mod(rng, 2, 32).astype(np.float32).astype(np.float64)
    ro = [0, 30, 64]
    exact = O.modulate(x, ro, mod)
    r = O.modulate_rounded(x, ro, mod, "bf16")
    rel = np.abs(r - exact) / np.maximum(np.abs(exact), 1e-30)
    assert np.all(rel <= 2.0 ** -8 + 1e-7)


def test_lookup_indexes_rows():
    tab = np.arange(5 * 3 * 2, dtype=np.float64).reshape(5, 3, 2)
    m = O.lookup(tab, [4, 0, 4])
    assert np.array_equal(m[0], tab[4]) and np.array_equal(m[1], tab[0])
    assert np.array_equal(m[2], tab[4])


# --------------------------------------------------------------------------- attention

def _brute_attention(q, k, v, ck, cv, Lc, ro, mod, H, hd, res):
    """Direct loops over the definition (independent of the vectorised oracle)."""
    n, D = len(q), len(q[0])
    beta = []
    for b in range(len(ro) - 1):
        beta += [b] * (ro[b + 1] - ro[b])
    keys = [list(ck[j]) for j in range(Lc)] + [list(k[j]) for j in range(n)]
    vals = [list(cv[j]) for j in range(Lc)] + [list(v[j]) for j in range(n)]
    out = [[0.0] * D for _ in range(n)]
    for i in range(n):
        b = beta[i]
        for h in range(H):
            qi = [q[i][h * hd + d] * (1.0 + mod[b][1][h * hd + d]) + mod[b][0][h * hd + d]
                  for d in range(hd)]
            s = []
            for key in keys:
                acc = 0.0
                for d in range(hd):
                    acc += qi[d] * key[h * hd + d]
                s.append(acc / math.sqrt(hd))
            m = max(s)
            e = [math.exp(x - m) for x in s]
            Z = sum(e)
            for d in range(hd):
                o = sum(e[j] * vals[j][h * hd + d] for j in range(len(keys))) / Z
                out[i][h * hd + d] = mod[b][2][h * hd + d] * o + res[i][h * hd + d]
    return np.array(out)


@pytest.mark.parametrize("Lc", [0, 2])
def test_attention_matches_brute_force_loops(Lc):
    rng = _rng(10 + Lc)
    H, hd, n = 2, 3, 5
    D = H * hd
    ro = [0, 2, 5]
    q, k, v = (rng.standard_normal((n, D)) for _ in range(3))
    ck = rng.standard_normal((3, D))
    cv = rng.standard_normal((3, D))
    ck[2:] = 1e30                     # beyond the valid length: must be ignored
    cv[2:] = np.nan
    mod = _mod(rng, 2, D)
    res = rng.standard_normal((n, D))
    got = O.window_attention(q, k, v, ck, cv, Lc, ro, mod, H, hd, residual=res)
    want = _brute_attention(q, k, v, ck, cv, Lc, ro, mod, H, hd, res)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)


def test_attention_two_keys_closed_form():
    # one query, one cached key and its own key: weights are sigmoid(s1 - s2)
    rng = _rng(20)
    hd = 8
    q = rng.standard_normal((1, hd))
    k = rng.standard_normal((1, hd))
    v = rng.standard_normal((1, hd))
    ck = rng.standard_normal((1, hd))
    cv = rng.standard_normal((1, hd))
    mod = _mod(rng, 1, hd, zero=True, gate_one=True)
    s1 = float(q[0] @ ck[0]) / math.sqrt(hd)
    s2 = float(q[0] @ k[0]) / math.sqrt(hd)
    w1 = 1.0 / (1.0 + math.exp(-(s1 - s2)))
    want = w1 * cv[0] + (1.0 - w1) * v[0]
    got = O.window_attention(q, k, v, ck, cv, 1, [0, 1], mod, 1, hd)
    np.testing.assert_allclose(got[0], want, rtol=0, atol=1e-14)


def test_attention_single_key_gives_gated_value():
    rng = _rng(21)
    D = 12
    q, k, v = (rng.standard_normal((1, D)) for _ in range(3))
    mod = _mod(rng, 1, D)
    got = O.window_attention(q, k, v, np.zeros((4, D)), np.zeros((4, D)), 0, [0, 1], mod, 3, 4)
    np.testing.assert_allclose(got[0], mod[0, 2] * v[0], rtol=0, atol=1e-15)


def test_attention_identical_keys_give_mean_of_values():
    rng = _rng(22)
    H, hd, n, Lc = 2, 4, 6, 3
    D = H * hd
    key = rng.standard_normal(D)
    k = np.tile(key, (n, 1))
    ck = np.tile(key, (Lc, 1))
    v = rng.standard_normal((n, D))
    cv = rng.standard_normal((Lc, D))
    q = rng.standard_normal((n, D))
    mod = _mod(rng, 2, D)
    mod[:, 2] = 1.0
    got = O.window_attention(q, k, v, ck, cv, Lc, [0, 2, 6], mod, H, hd)
    want = np.concatenate([cv, v]).mean(axis=0)
    np.testing.assert_allclose(got, np.tile(want, (n, 1)), rtol=0, atol=1e-14)


def test_attention_values_one_give_gate():
    # probabilities sum to one in every row
    rng = _rng(23)
    H, hd, n, Lc = 3, 4, 7, 5
    D = H * hd
    q, k = (rng.standard_normal((n, D)) * 3 for _ in range(2))
    ck = rng.standard_normal((Lc, D)) * 3
    mod = _mod(rng, 3, D)
    got = O.window_attention(q, k, np.ones((n, D)), ck, np.ones((Lc, D)), Lc, [0, 1, 4, 7],
                             mod, H, hd)
    beta = O.row_blocks([0, 1, 4, 7], n)
    np.testing.assert_allclose(got, mod[beta, 2], rtol=0, atol=1e-14)


@pytest.mark.parametrize("Lc", [0, 9])
def test_attention_reduces_to_torch_sdpa(Lc):
    # empty or non-empty cache, one shared timestep, zero shift/scale, gate 1:
    # plain full attention over [cache ; window]
    torch.manual_seed(24)
    H, hd, n = 4, 16, 33
    D = H * hd
    q, k, v = (torch.randn(n, D, dtype=torch.float64) for _ in range(3))
    ck, cv = (torch.randn(Lc, D, dtype=torch.float64) for _ in range(2))
    mod = np.zeros((1, 3, D))
    mod[0, 2] = 1.0
    got = O.window_attention(q, k, v, ck, cv, Lc, [0, n], mod, H, hd)
    K = torch.cat([ck, k]).view(-1, H, hd).transpose(0, 1)[None]
    V = torch.cat([cv, v]).view(-1, H, hd).transpose(0, 1)[None]
    Q = q.view(n, H, hd).transpose(0, 1)[None]
    want = torch.nn.functional.scaled_dot_product_attention(Q, K, V)
    want = want[0].transpose(0, 1).reshape(n, D).numpy()
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_attention_permutation_invariance():
    # permute rows inside each block and the order of the blocks (moving their
    # adaLN rows with them), and the cache rows: outputs permute the same way
    rng = _rng(25)
    H, hd = 2, 8
    D = H * hd
    sizes = [3, 5, 4]
    ro = [0, 3, 8, 12]
    n, Lc = 12, 6
    q, k, v = (rng.standard_normal((n, D)) for _ in range(3))
    ck, cv = (rng.standard_normal((Lc, D)) for _ in range(2))
    mod = _mod(rng, 3, D)
    base = O.window_attention(q, k, v, ck, cv, Lc, ro, mod, H, hd)
    border = [2, 0, 1]
    perm = []
    new_ro = [0]
    for b in border:
        rows = list(range(ro[b], ro[b + 1]))
        rng.shuffle(rows)
        perm += rows
        new_ro.append(new_ro[-1] + sizes[b])
    perm = np.array(perm)
    cperm = rng.permutation(Lc)
    got = O.window_attention(q[perm], k[perm], v[perm], ck[cperm], cv[cperm], Lc, new_ro,
                             mod[border], H, hd)
    np.testing.assert_allclose(got, base[perm], rtol=0, atol=1e-12)


def test_attention_gate_zero_returns_residual():
    rng = _rng(26)
    n, D = 5, 8
    q, k, v, res = (rng.standard_normal((n, D)) for _ in range(4))
    mod = _mod(rng, 1, D)
    mod[0, 2] = 0.0
    got = O.window_attention(q, k, v, np.zeros((0, D)), np.zeros((0, D)), 0, [0, n], mod, 2, 4,
                             residual=res)
    assert np.array_equal(got, res)


def test_attention_rows_subset_matches_full():
    rng = _rng(27)
    n, D = 40, 16
    q, k, v = (rng.standard_normal((n, D)) for _ in range(3))
    ck, cv = (rng.standard_normal((7, D)) for _ in range(2))
    mod = _mod(rng, 2, D)
    full = O.window_attention(q, k, v, ck, cv, 7, [0, 17, 40], mod, 2, 8, q_chunk=8)
    rows = [39, 0, 16, 17]
    sub = O.window_attention(q, k, v, ck, cv, 7, [0, 17, 40], mod, 2, 8, rows=rows)
    np.testing.assert_allclose(sub, full[rows], rtol=0, atol=1e-14)


def test_window_step_modulates_k_and_v_with_their_blocks():
    rng = _rng(28)
    n, D = 9, 8
    q, k, v = (rng.standard_normal((n, D)) for _ in range(3))
    mod = _mod(rng, 2, D)
    mod[:, 1] = -1.0                      # k' = v' = shift of the row's block
    out, kp, vp = O.window_step(q, k, v, np.zeros((0, D)), np.zeros((0, D)), 0, [0, 4, 9],
                                mod, 2, 4)
    for i in range(n):
        b = 0 if i < 4 else 1
        assert np.array_equal(kp[i], mod[b, 0]) and np.array_equal(vp[i], mod[b, 0])


# --------------------------------------------------------------------------- queue and cache

def test_cache_after_k_advances_holds_kth_exited_block():
    rng = _rng(30)
    D = 6
    c = O.KVCacheRing(1, 10, D)
    exits = []
    for a in range(5):
        n = [10, 7, 10, 3, 10][a]
        ke, ve = rng.standard_normal((n, D)), rng.standard_normal((n, D))
        exits.append((ke, ve, n))
        c.advance(ke, ve, n)
        k, v, L = c.latest()
        assert L == n and np.array_equal(k[:n], ke) and np.array_equal(v[:n], ve)
        assert c.n_advances == a + 1
    with pytest.raises(ValueError):
        c.advance(np.zeros((11, D)), np.zeros((11, D)), 11)


def test_cache_ring_slot_rotation():
    c = O.KVCacheRing(3, 4, 2)
    slots = [c.advance(np.full((4, 2), a), np.full((4, 2), -a), 4) for a in range(7)]
    assert slots == [0, 1, 2, 0, 1, 2, 0]
    assert np.all(c.k[0] == 6) and np.all(c.k[1] == 4) and np.all(c.k[2] == 5)


def test_fifo_queue_order_and_window():
    q = O.FifoQueue(3)
    for i in range(3):
        q.push(np.full((2 + i, 2), i))
    with pytest.raises(ValueError):
        q.push(np.zeros((2, 2)))
    assert q.row_offset() == [0, 2, 5, 9]
    assert q.pop().ident == 0
    q.push(np.full((1, 2), 3))
    assert [b.ident for b in q.blocks] == [1, 2, 3]
    assert np.array_equal(q.window()[:, 0], [1, 1, 1, 2, 2, 2, 2, 3])


# --------------------------------------------------------------------------- long-run schedule

def test_timestep_schedule_matches_linspace():
    tau = O.timestep_schedule(50)
    assert tau == [int(x) for x in np.round(np.linspace(999, 0, 50))]
    assert tau[0] == 999 and tau[-1] == 0 and all(a > b for a, b in zip(tau, tau[1:]))


@pytest.mark.parametrize("n_blocks,W,T", [(129, 8, 50), (10, 3, 7), (5, 4, 4)])
def test_long_run_schedule_invariants(n_blocks, W, T):
    sch = O.long_run_schedule(n_blocks, W, T)
    evals = {b: [] for b in range(n_blocks)}
    pops, pushes = [], []
    for st in sch:
        assert 1 <= len(st["live"]) <= W
        assert st["live"] == sorted(st["live"])                       # FIFO order
        assert all(a > b for a, b in zip(st["k"], st["k"][1:]))      # head cleanest
        for b, k in zip(st["live"], st["k"]):
            evals[b].append((st["step"], k))
        pops += st["pop_after"]
        pushes += st["push_after"]
        for b in st["pop_after"]:
            if b + W < n_blocks and st["step"] + 1 < len(sch):
                assert b + W in st["push_after"]                    # one in, one out
    for b, ev in evals.items():
        assert [k for _, k in ev] == list(range(T))                  # T evaluations in order
        assert [s for s, _ in ev] == list(range(ev[0][0], ev[0][0] + T))
    assert pops == list(range(n_blocks))
    assert pushes == list(range(1, n_blocks))
    assert len(sch) == (n_blocks - 1) * T // W + T


def test_long_run_config_shape():
    from workloads import run_config
    rc = run_config()
    rows = rc.block_rows
    assert len(rows) == 129 and rows[-1] == 1350 and all(r == 2700 for r in rows[:-1])
    sch = O.long_run_schedule(len(rows), rc.window_blocks, rc.n_timesteps)
    assert len(sch) == 850
    assert max(len(s["live"]) for s in sch) == 8


def test_long_run_oracle_cache_follows_exits():
    rng = _rng(31)
    D, H, hd = 8, 2, 4
    noise = [rng.standard_normal((r, D)) for r in [4, 4, 4, 4, 2]]
    table = np.tanh(rng.standard_normal((1000, 3, D)))
    run = O.LongRun(noise, table, H, hd, window_blocks=2, n_timesteps=3)
    # entries floor(b * 3 / 2) = 0, 1, 3, 4, 6; block 0 exits after step 2
    x, ro, t, mod, ck, cv, L = run.step_inputs(2)
    assert L == 0 and ro == [0, 4, 8] and t == [run.tau[2], run.tau[1]]
    x, ro, t, mod, ck, cv, L = run.step_inputs(3)
    assert L == 4
    want = O.modulate(noise[0], [0, 4], O.lookup(table, [run.tau[2]]))
    assert np.array_equal(ck, want)
    assert np.array_equal(x[:4], noise[1])


def test_long_run_schedule_golden():
    import collections
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "long_run_schedule.json")
    with open(path) as f:
        g = json.load(f)
    sch = O.long_run_schedule(129, 8, 50)
    hist = collections.Counter(len(s["live"]) for s in sch)
    # hand-derived: warm-up and cool-down each pass through 1..7 live blocks
    assert {str(k): v for k, v in sorted(hist.items())} == g["block_count_histogram"]
    assert g["block_count_histogram"] == {"1": 13, "2": 12, "3": 12, "4": 13, "5": 13,
                                          "6": 12, "7": 12, "8": 763}
    assert len(sch) == g["n_steps"] == 850
    assert [O.entry_step(b, 50, 8) for b in range(10)] == g["entry_steps_first_10"]
    assert [s["step"] for s in sch if s["pop_after"]][:3] == g["pop_steps_first_3"]
    assert O.timestep_schedule(50)[:5] == g["tau_first_5"]


def test_long_run_context_of_several_exited_blocks():
    """context_blocks = C: the cache is the K'/V' of the last C exited blocks (each modulated at
    the last timestep); C = 1 is the single exited block of the default run."""
    rng = np.random.default_rng(5)
    D, rows = 8, [6, 6, 6, 6, 6, 3]
    noise = [rng.standard_normal((r, D)) for r in rows]
    table = np.tanh(rng.standard_normal((1000, 3, D)))
    one = O.LongRun(noise, table, 2, 4, window_blocks=2, n_timesteps=4)
    three = O.LongRun(noise, table, 2, 4, window_blocks=2, n_timesteps=4, context_blocks=3)
    m_last = O.lookup(table, [O.timestep_schedule(4)[3]])
    for s in range(len(one.schedule)):
        exited = [b for b in range(len(noise)) if any(b in one.schedule[u]["pop_after"] for u in range(s))]
        _, _, _, _, ck1, _, L1 = one.step_inputs(s)
        _, _, _, _, ck3, _, L3 = three.step_inputs(s)
        assert L1 == (rows[exited[-1]] if exited else 0)
        assert L3 == sum(rows[b] for b in exited[-3:])
        want = [O.modulate(noise[b], [0, rows[b]], m_last) for b in exited[-3:]]
        assert np.array_equal(ck3, np.concatenate(want) if want else np.zeros((0, D)))
        if exited:
            assert np.array_equal(ck1, want[-1])

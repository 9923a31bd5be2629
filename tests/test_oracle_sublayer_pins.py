"""Pins of the sublayer oracle (oracle/sublayer.py) to things other than itself: hand-computed
values, closed forms, brute-force loops on tiny inputs, and the reduction of the whole
sublayer to the already pinned window attention when the projections are identities.
A final check plants one mistake at a time in the oracle (on the CPU) and requires that
some pin fails for each."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import oracle.sublayer as S


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _mod(n_blocks, D, seed):
    return np.tanh(_rand((n_blocks, 3, D), seed))


# ----------------------------------------------------------------------------- pins

def pin_round_to_hand_cases():
    # bf16 keeps 8 significand bits: 1 + 2^-8 is a tie -> even (1.0); 1 + 3 * 2^-9 -> 1 + 2^-7
    got = S.round_to(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -9, -2.5]), "bf16")
    assert list(got) == [1.0, 1 + 2.0 ** -7, -2.5]
    # f16 keeps 11 bits: 1 + 2^-11 is a tie -> 1.0; beyond 65504 saturates
    got = S.round_to(np.array([1 + 2.0 ** -11, 1 + 3 * 2.0 ** -12, 70000.0, -1e6]), "f16")
    assert list(got) == [1.0, 1 + 2.0 ** -10, 65504.0, -65504.0]


def pin_layer_norm_hand_row():
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    got = S.layer_norm(x, 1e-6)
    want = (x - 2.5) / math.sqrt(1.25 + 1e-6)      # biased variance: (2.25+0.25+0.25+2.25)/4
    assert np.allclose(got, want, rtol=0, atol=1e-15)


def pin_layer_norm_moments_and_constant_rows():
    x = _rand((7, 96), 1, 3.0) + 5.0
    eps = 1e-3
    y = S.layer_norm(x, eps)
    v = x.var(axis=1)
    assert np.allclose(y.mean(axis=1), 0.0, atol=1e-12)
    assert np.allclose((y * y).mean(axis=1), v / (v + eps), rtol=1e-12)
    assert np.array_equal(S.layer_norm(np.full((2, 8), 3.25), 1e-6), np.zeros((2, 8)))


def pin_layer_norm_brute_force():
    x = _rand((3, 5), 2)
    eps = 0.01
    y = S.layer_norm(x, eps)
    for i in range(3):
        mean = sum(x[i]) / 5
        var = sum((x[i, c] - mean) ** 2 for c in range(5)) / 5
        for c in range(5):
            assert abs(y[i, c] - (x[i, c] - mean) / math.sqrt(var + eps)) < 1e-13


def pin_ln_modulate_special_cases():
    x = _rand((6, 8), 3)
    ro = [0, 2, 6]
    zero = np.zeros((2, 3, 8))
    assert np.array_equal(S.ln_modulate(x, ro, zero, 1e-6), S.layer_norm(x, 1e-6))
    mod = _mod(2, 8, 4)
    mod[:, 1, :] = -1.0                              # scale -1: every row becomes its block's shift
    got = S.ln_modulate(x, ro, mod, 1e-6)
    assert np.array_equal(got[:2], np.broadcast_to(mod[0, 0], (2, 8)))
    assert np.array_equal(got[2:], np.broadcast_to(mod[1, 0], (4, 8)))
    mod = _mod(2, 8, 5)                              # a hand-built row of block 1
    n = S.layer_norm(x, 1e-6)
    assert np.allclose(S.ln_modulate(x, ro, mod, 1e-6)[3], n[3] * (1 + mod[1, 1]) + mod[1, 0], atol=1e-15)


def pin_linear_brute_force_and_identity():
    a, w, b = _rand((3, 4), 6), _rand((5, 4), 7), _rand(5, 8)
    y = S.linear(a, w, b)
    for i in range(3):
        for j in range(5):
            assert abs(y[i, j] - (sum(a[i, c] * w[j, c] for c in range(4)) + b[j])) < 1e-13
    assert np.allclose(S.linear(a, np.eye(4), np.arange(4.0)), a + np.arange(4.0), atol=1e-15)


def _identity_case(seed=9, Lc=3):
    H, hd = 2, 4
    D = H * hd
    ro = [0, 3, 7]
    x = _rand((7, D), seed)
    ck, cv = _rand((4, D), seed + 1), _rand((4, D), seed + 2)
    mod = _mod(2, D, seed + 3)
    return H, hd, D, ro, x, ck, cv, mod, Lc


def pin_sublayer_identity_projections_reduce_to_window_attention():
    H, hd, D, ro, x, ck, cv, mod, Lc = _identity_case()
    eye = np.eye(D)
    w_qkv = np.concatenate([eye, eye, eye], axis=0)
    out, k, v = S.sublayer_step(x, w_qkv, None, eye, None, ck, cv, Lc, ro, mod, H, hd, 1e-6, rounded=False)
    h = S.ln_modulate(x, ro, mod, 1e-6)
    want = O.window_attention(h, h, h, ck, cv, Lc, ro, mod, H, hd, mod_q=False, gate_out=True, residual=x)
    assert np.allclose(out, want, rtol=0, atol=1e-12)
    assert np.array_equal(k, h) and np.array_equal(v, h)


def _brute_sublayer(x, w_qkv, b_qkv, w_o, b_o, ck, cv, Lc, ro, mod, H, hd, eps):
    n, D = x.shape
    beta = [next(b for b in range(len(ro) - 1) if ro[b] <= i < ro[b + 1]) for i in range(n)]
    h = np.zeros((n, D))
    for i in range(n):
        mean = sum(x[i]) / D
        var = sum((x[i, c] - mean) ** 2 for c in range(D)) / D
        for c in range(D):
            h[i, c] = (x[i, c] - mean) / math.sqrt(var + eps) * (1 + mod[beta[i], 1, c]) + mod[beta[i], 0, c]
    qkv = np.zeros((n, 3 * D))
    for i in range(n):
        for j in range(3 * D):
            qkv[i, j] = sum(h[i, c] * w_qkv[j, c] for c in range(D)) + b_qkv[j]
    q, k, v = qkv[:, :D], qkv[:, D:2 * D], qkv[:, 2 * D:]
    K = [ck[j] for j in range(Lc)] + [k[j] for j in range(n)]
    V = [cv[j] for j in range(Lc)] + [v[j] for j in range(n)]
    o = np.zeros((n, D))
    for i in range(n):
        for hh in range(H):
            sl = slice(hh * hd, (hh + 1) * hd)
            s = [sum(q[i, sl] * K[j][sl]) / math.sqrt(hd) for j in range(len(K))]
            m = max(s)
            e = [math.exp(t - m) for t in s]
            z = sum(e)
            for d in range(hd):
                o[i, hh * hd + d] = sum(e[j] * V[j][hh * hd + d] for j in range(len(K))) / z
    out = np.zeros((n, D))
    for i in range(n):
        for j in range(D):
            out[i, j] = x[i, j] + mod[beta[i], 2, j] * (sum(o[i, c] * w_o[j, c] for c in range(D)) + b_o[j])
    return out, k, v


def pin_sublayer_brute_force_loops():
    H, hd, D, ro, x, ck, cv, mod, Lc = _identity_case(seed=11)
    w_qkv, b_qkv = _rand((3 * D, D), 20, 0.4), _rand(3 * D, 21, 0.1)
    w_o, b_o = _rand((D, D), 22, 0.4), _rand(D, 23, 0.1)
    want, wk, wv = _brute_sublayer(x, w_qkv, b_qkv, w_o, b_o, ck, cv, Lc, ro, mod, H, hd, 1e-5)
    got, k, v = S.sublayer_step(x, w_qkv, b_qkv, w_o, b_o, ck, cv, Lc, ro, mod, H, hd, 1e-5, rounded=False)
    assert np.allclose(got, want, rtol=0, atol=1e-12)
    assert np.allclose(k, wk, atol=1e-12) and np.allclose(v, wv, atol=1e-12)
    rows = [6, 0, 3]
    got_rows, _, _ = S.sublayer_step(x, w_qkv, b_qkv, w_o, b_o, ck, cv, Lc, ro, mod, H, hd, 1e-5,
                                     rounded=False, rows=rows)
    assert np.allclose(got_rows, want[rows], rtol=0, atol=1e-12)


def pin_sublayer_rounded_stores_16_bit_intermediates():
    H, hd, D, ro, x, ck, cv, mod, Lc = _identity_case(seed=13)
    w_qkv, b_qkv = _rand((3 * D, D), 30, 0.4), _rand(3 * D, 31, 0.1)
    w_o, b_o = _rand((D, D), 32, 0.4), _rand(D, 33, 0.1)
    _, k, v = S.sublayer_step(x, w_qkv, b_qkv, w_o, b_o, ck, cv, Lc, ro, mod, H, hd, 1e-6, rounded=True)
    h = S.round_to(S.ln_modulate(x, ro, mod, 1e-6), "bf16")
    kk = S.linear(h, w_qkv, b_qkv)[:, D:2 * D]
    assert np.array_equal(k, S.round_to(kk, "f16"))
    assert np.array_equal(np.asarray(torch.from_numpy(k).to(torch.float16).to(torch.float64)), k)


PINS = [pin_round_to_hand_cases, pin_layer_norm_hand_row, pin_layer_norm_moments_and_constant_rows,
        pin_layer_norm_brute_force, pin_ln_modulate_special_cases, pin_linear_brute_force_and_identity,
        pin_sublayer_identity_projections_reduce_to_window_attention, pin_sublayer_brute_force_loops,
        pin_sublayer_rounded_stores_16_bit_intermediates]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# ----------------------------------------------------------------------------- planted mistakes

def _mutants():
    ln, lnm, lin, step, rnd = S.layer_norm, S.ln_modulate, S.linear, S.sublayer_step, S.round_to

    def ln_unbiased(x, eps):
        x = O.as_f64(x)
        d = x - x.mean(axis=1, keepdims=True)
        return d / np.sqrt(d.var(axis=1, ddof=1, keepdims=True) + eps)

    def ln_eps_outside(x, eps):
        x = O.as_f64(x)
        d = x - x.mean(axis=1, keepdims=True)
        return d / (np.sqrt((d * d).mean(axis=1, keepdims=True)) + eps)

    def lnm_scale_not_plus_one(x, ro, mod, eps):
        n = S.layer_norm(x, eps)
        m = O.as_f64(mod)
        b = O.row_blocks(ro, n.shape[0])
        return n * m[b, 1, :] + m[b, 0, :]

    def lnm_shift_scale_swapped(x, ro, mod, eps):
        n = S.layer_norm(x, eps)
        m = O.as_f64(mod)
        b = O.row_blocks(ro, n.shape[0])
        return n * (1.0 + m[b, 0, :]) + m[b, 1, :]

    def lin_no_bias(a, w, bias=None):
        return lin(a, w, None)

    def lin_transposed(a, w, bias=None):
        y = O.as_f64(a) @ O.as_f64(w)[:, :O.as_f64(a).shape[1]].T[:, ::-1]
        return y if bias is None else y + O.as_f64(bias)[None, :]

    def step_qk_swapped(x, w_qkv, b_qkv, w_o, b_o, ck, cv, Lc, ro, mod, H, hd, eps, *, rounded=True, rows=None):
        D = O.as_f64(x).shape[1]
        w = O.as_f64(w_qkv)
        w2 = np.concatenate([w[D:2 * D], w[:D], w[2 * D:]], axis=0)
        b2 = None if b_qkv is None else np.concatenate([O.as_f64(b_qkv)[D:2 * D], O.as_f64(b_qkv)[:D],
                                                        O.as_f64(b_qkv)[2 * D:]])
        return step(x, w2, b2, w_o, b_o, ck, cv, Lc, ro, mod, H, hd, eps, rounded=rounded, rows=rows)

    def step_no_gate(x, w_qkv, b_qkv, w_o, b_o, ck, cv, Lc, ro, mod, H, hd, eps, *, rounded=True, rows=None):
        m = O.as_f64(mod).copy()
        out, k, v = step(x, w_qkv, b_qkv, w_o, b_o, ck, cv, Lc, ro, m, H, hd, eps, rounded=rounded, rows=rows)
        sel = np.arange(O.as_f64(x).shape[0]) if rows is None else np.asarray(rows)
        beta = O.row_blocks(ro, O.as_f64(x).shape[0])[sel]
        g = m[beta, 2, :]
        return O.as_f64(x)[sel] + (out - O.as_f64(x)[sel]) / np.where(g == 0, 1, g), k, v

    def step_no_residual(x, *args, rounded=True, rows=None):
        out, k, v = step(x, *args, rounded=rounded, rows=rows)
        sel = np.arange(O.as_f64(x).shape[0]) if rows is None else np.asarray(rows)
        return out - O.as_f64(x)[sel], k, v

    def step_cache_dropped(x, w_qkv, b_qkv, w_o, b_o, ck, cv, Lc, ro, mod, H, hd, eps, *, rounded=True, rows=None):
        return step(x, w_qkv, b_qkv, w_o, b_o, ck, cv, 0, ro, mod, H, hd, eps, rounded=rounded, rows=rows)

    def rnd_truncate(x, dtype):
        import torch
        t = torch.from_numpy(np.ascontiguousarray(O.as_f64(x))).to(torch.float32)
        bits = t.view(torch.int32)
        keep = 16 if dtype == "bf16" else 13
        if dtype == "f32":
            return rnd(x, dtype)
        t2 = (bits & ~((1 << keep) - 1)).view(torch.float32)
        return rnd(t2.to(torch.float64).numpy(), dtype)

    return [("layer_norm", ln_unbiased), ("layer_norm", ln_eps_outside),
            ("ln_modulate", lnm_scale_not_plus_one), ("ln_modulate", lnm_shift_scale_swapped),
            ("linear", lin_no_bias), ("linear", lin_transposed),
            ("sublayer_step", step_qk_swapped), ("sublayer_step", step_no_gate),
            ("sublayer_step", step_no_residual), ("sublayer_step", step_cache_dropped),
            ("round_to", rnd_truncate)]


@pytest.mark.parametrize("idx", range(11))
def test_planted_mistake_fails_a_pin(idx, monkeypatch):
    name, fn = _mutants()[idx]
    monkeypatch.setattr(S, name, fn)
    failed = []
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake in {name} ({fn.__name__})"

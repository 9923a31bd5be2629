"""Pins of the fresh-context oracle (oracle/context.py) to things other than itself: the
features the already pinned window step and sublayer step produce for the same rows, a
hand-computed closed form, the long run's cache at its final timestep, and planted mistakes
(one at a time, on the CPU), each of which must fail some pin."""
import math

import numpy as np
import pytest

import oracle as O
import oracle.context as C
import oracle.sublayer as S


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _mod(n_blocks, D, seed):
    return np.tanh(_rand((n_blocks, 3, D), seed))


def pin_fresh_equals_window_step_features():
    # the window step's own k', v' of a block's rows, recomputed from those rows alone
    H, hd = 2, 4
    D = H * hd
    ro = [0, 3, 7]
    q, k, v = _rand((7, D), 1), _rand((7, D), 2), _rand((7, D), 3)
    mod = _mod(2, D, 4)
    _, kp, vp = O.window_step(q, k, v, np.zeros((0, D)), np.zeros((0, D)), 0, ro, mod, H, hd)
    for b in range(2):
        r0, r1 = ro[b], ro[b + 1]
        fk, fv = C.fresh_context(k[r0:r1], v[r0:r1], [0, r1 - r0], mod[b:b + 1])
        assert np.array_equal(fk, kp[r0:r1]) and np.array_equal(fv, vp[r0:r1])
    # a context of two blocks at once
    fk, fv = C.fresh_context(k, v, ro, mod)
    assert np.array_equal(fk, kp) and np.array_equal(fv, vp)


def pin_fresh_identity_special_cases():
    x = _rand((5, 8), 5)
    zero = np.zeros((1, 3, 8))
    fk, fv = C.fresh_context(x, 2 * x, [0, 5], zero)
    assert np.array_equal(fk, x) and np.array_equal(fv, 2 * x)
    mod = _mod(1, 8, 6)
    mod[0, 1, :] = -1.0                        # scale -1: every row becomes the shift
    fk, _ = C.fresh_context(x, x, [0, 5], mod)
    assert np.array_equal(fk, np.broadcast_to(mod[0, 0], (5, 8)))


def pin_fresh_sublayer_equals_step_features():
    # the sublayer step's projected k, v of a block's rows, recomputed from those rows alone
    H, hd = 2, 4
    D = H * hd
    ro = [0, 3, 7]
    x = _rand((7, D), 7)
    mod = _mod(2, D, 8)
    w_qkv, b_qkv = _rand((3 * D, D), 9, 0.4), _rand(3 * D, 10, 0.1)
    w_o, b_o = _rand((D, D), 11, 0.4), _rand(D, 12, 0.1)
    for rounded in (False, True):
        _, k, v = S.sublayer_step(x, w_qkv, b_qkv, w_o, b_o, np.zeros((0, D)), np.zeros((0, D)), 0, ro, mod,
                                  H, hd, 1e-5, rounded=rounded)
        for b in range(2):
            r0, r1 = ro[b], ro[b + 1]
            fk, fv = C.fresh_context_sublayer(x[r0:r1], [0, r1 - r0], mod[b:b + 1], w_qkv, b_qkv, 1e-5,
                                              rounded=rounded)
            assert np.array_equal(fk, k[r0:r1]) and np.array_equal(fv, v[r0:r1])


def pin_fresh_sublayer_closed_form():
    # x = (1, 2, 3, 4): mean 5/2, biased variance 5/4; with eps = 1/4, LN(x) = (x - 5/2) / sqrt(3/2)
    # = (-sqrt(3/2), -sqrt(1/6), sqrt(1/6), sqrt(3/2)).  W_k = I with b_k = (1/2, 0, 0, 0), W_v = 2 I.
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    eye = np.eye(4)
    w_qkv = np.concatenate([np.full((4, 4), 7.0), eye, 2 * eye], axis=0)
    b_qkv = np.array([9.0, 9.0, 9.0, 9.0, 0.5, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0])
    k, v = C.fresh_context_sublayer(x, [0, 1], np.zeros((1, 3, 4)), w_qkv, b_qkv, 0.25, rounded=False)
    a, c = 1.2247448713915890, 0.4082482904638631          # sqrt(3/2), sqrt(1/6)
    assert np.allclose(k, [[-a + 0.5, -c, c, a]], rtol=0, atol=1e-15)
    assert np.allclose(v, [[-2 * a, -2 * c, 2 * c, 2 * a]], rtol=0, atol=1e-15)


def pin_long_run_cache_is_fresh_at_the_final_timestep():
    # The long run's cache is the exited block's features from its last evaluation, at the
    # schedule's final timestep (0).  Recomputed with the conditioning of timestep 0 they are
    # the same: with the latents not updated, the two variants differ only in their cost.
    H, hd, rows = 2, 4, 6
    D = H * hd
    noise = [_rand((rows, D), 20 + b) for b in range(4)]
    table = np.tanh(_rand((1000, 3, D), 30))
    run = O.LongRun(noise, table, H, hd, window_blocks=2, n_timesteps=4)
    tau = O.timestep_schedule(4)
    assert tau[-1] == 0
    for s in range(len(run.schedule)):
        _, _, _, _, ck, cv, L = run.step_inputs(s)
        exited = [b for b in range(4) if any(b in run.schedule[u]["pop_after"] for u in range(s))]
        if not exited:
            assert L == 0
            continue
        lat = noise[exited[-1]]
        fk, fv = C.fresh_context(lat, lat, [0, rows], O.lookup(table, [0]))
        assert L == rows and np.array_equal(ck, fk) and np.array_equal(cv, fv)
        # conditioned on another timestep, the recomputed features differ
        gk, _ = C.fresh_context(lat, lat, [0, rows], O.lookup(table, [500]))
        assert not np.allclose(gk, ck)


PINS = [pin_fresh_equals_window_step_features, pin_fresh_identity_special_cases,
        pin_fresh_sublayer_equals_step_features, pin_fresh_sublayer_closed_form,
        pin_long_run_cache_is_fresh_at_the_final_timestep]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


def _mutants():
    fc, fs = C.fresh_context, C.fresh_context_sublayer

    def fc_ignores_mod(k_ctx, v_ctx, ro, mod):
        return O.as_f64(k_ctx), O.as_f64(v_ctx)

    def fc_scale_not_plus_one(k_ctx, v_ctx, ro, mod):
        m = O.as_f64(mod)
        b = O.row_blocks(ro, O.as_f64(k_ctx).shape[0])
        return (O.as_f64(k_ctx) * m[b, 1] + m[b, 0], O.as_f64(v_ctx) * m[b, 1] + m[b, 0])

    def fc_k_for_v(k_ctx, v_ctx, ro, mod):
        k, _ = fc(k_ctx, v_ctx, ro, mod)
        return k, k

    def fs_q_rows_for_k(x_ctx, ro, mod, w_qkv, b_qkv, eps, *, rounded=True):
        w, b = O.as_f64(w_qkv), O.as_f64(b_qkv)
        D = O.as_f64(x_ctx).shape[1]
        w2 = np.concatenate([w[:D], w[:D], w[2 * D:]], axis=0)
        b2 = np.concatenate([b[:D], b[:D], b[2 * D:]])
        return fs(x_ctx, ro, mod, w2, b2, eps, rounded=rounded)

    def fs_k_v_swapped(x_ctx, ro, mod, w_qkv, b_qkv, eps, *, rounded=True):
        k, v = fs(x_ctx, ro, mod, w_qkv, b_qkv, eps, rounded=rounded)
        return v, k

    def fs_no_bias(x_ctx, ro, mod, w_qkv, b_qkv, eps, *, rounded=True):
        return fs(x_ctx, ro, mod, w_qkv, None, eps, rounded=rounded)

    def fs_no_layer_norm(x_ctx, ro, mod, w_qkv, b_qkv, eps, *, rounded=True):
        x = O.as_f64(x_ctx)
        D = x.shape[1]
        h = O.modulate(x, ro, mod)
        w, b = O.as_f64(w_qkv), O.as_f64(b_qkv)
        k, v = S.linear(h, w[D:2 * D], b[D:2 * D]), S.linear(h, w[2 * D:], b[2 * D:])
        return (S.round_to(k, "f16"), S.round_to(v, "f16")) if rounded else (k, v)

    def fs_unrounded_h(x_ctx, ro, mod, w_qkv, b_qkv, eps, *, rounded=True):
        k, v = fs(x_ctx, ro, mod, w_qkv, b_qkv, eps, rounded=False)
        return (S.round_to(k, "f16"), S.round_to(v, "f16")) if rounded else (k, v)

    return [("fresh_context", fc_ignores_mod), ("fresh_context", fc_scale_not_plus_one),
            ("fresh_context", fc_k_for_v), ("fresh_context_sublayer", fs_q_rows_for_k),
            ("fresh_context_sublayer", fs_k_v_swapped), ("fresh_context_sublayer", fs_no_bias),
            ("fresh_context_sublayer", fs_no_layer_norm), ("fresh_context_sublayer", fs_unrounded_h)]


@pytest.mark.parametrize("idx", range(8))
def test_planted_mistake_fails_a_pin(idx, monkeypatch):
    name, fn = _mutants()[idx]
    monkeypatch.setattr(C, name, fn)
    failed = []
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake in {name} ({fn.__name__})"

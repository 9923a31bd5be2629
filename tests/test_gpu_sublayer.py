"""GPU parity of the DiT attention sublayer (pre-norm with adaLN modulation, q/k/v and output
projections on the tensor cores, gated residual, and the sublayer step with its advance)
against the float64 oracle on the same seeded inputs, through the C ABI.

Bounds: a 16-bit store of a value v is within one unit in the last place of v (2^-8 |v|
for bf16, 2^-11 |v| for f16); a fp32 dot product of k terms is within k * 2^-24 times the
sum of |terms|, at most 2^-12 times it for the k <= 4096 used here.  The whole step is held
to the bf16 bar of the window step, max-abs 2e-2 and relative L2 5e-3, twice: against the
plain float64 definition (no intermediate rounded) and against the oracle that stores its
intermediates where the kernels do (h, q, o bf16; k, v f16)."""
import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import assert_close, bytes_equal, errors, sample_rows
from workloads import as_features, make_step_inputs, make_sublayer_weights, step_config

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

EPS = 1e-6


def _table(D, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.tanh(torch.randn(1000, 3, D, generator=g))


def _bf16(shape, seed, std=1.0, mean=0.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * std + mean).to(torch.bfloat16)


def _dot_bound(a, w):
    """fp32 accumulation error bound of a W^T: 2^-12 * sum_c |a_c| |w_c| (k <= 4096 terms)."""
    assert a.shape[1] <= 4096
    return (np.abs(a) @ np.abs(w).T) * 2.0 ** -12


@pytest.mark.parametrize("D,rows", [(256, [300, 211]), (1536, [129, 128, 1]), (3072, [64, 300])])
def test_ln_modulate_matches_oracle(dp, D, rows):
    x = _bf16((sum(rows), D), 1, std=2.0, mean=0.5)
    table = _table(D, 2)
    ts = [7, 500, 999][:len(rows)]
    blk = dp.blocks_from_table(table.cuda(), ts, rows)
    h = torch.empty_like(x, device="cuda")
    dp.ln_modulate(x.cuda(), h, blk, EPS)
    dp.device_status()
    want = O.ln_modulate(x, np.cumsum([0] + rows), O.lookup(table, ts), EPS)
    got = h.cpu().double().numpy()
    # one bf16 rounding of a value computed in fp32 (its error far below one bf16 unit)
    assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-6)
    assert np.mean(got == O.round_to(want, "bf16")) > 0.99


@pytest.mark.parametrize("m,n,k,ydt", [(300, 256, 512, torch.bfloat16), (257, 384, 200, torch.float16),
                                       (128, 128, 64, torch.bfloat16), (1000, 512, 3072, torch.float16)])
def test_linear_matches_oracle(dp, m, n, k, ydt):
    a = _bf16((m, k), 3)
    w = _bf16((n, k), 4, std=k ** -0.5)
    bias = torch.randn(n, generator=torch.Generator().manual_seed(5)) * 0.1
    y = torch.empty(m, n, dtype=ydt, device="cuda")
    dp.linear(a.cuda(), w.cuda(), bias.cuda(), y)
    dp.device_status()
    exact = O.linear(a, w, bias)
    got = y.cpu().double().numpy()
    unit = 2.0 ** -8 if ydt == torch.bfloat16 else 2.0 ** -11
    bound = unit * np.abs(exact) + _dot_bound(O.as_f64(a), O.as_f64(w)) + 1e-7
    assert np.all(np.abs(got - exact) <= bound), float(np.max(np.abs(got - exact) - bound))


def test_qkv_project_splits_q_k_v(dp):
    D, m = 512, 333
    h = _bf16((m, D), 6)
    wts = make_sublayer_weights(D, 7)
    q = torch.empty(m, D, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(m, D, dtype=torch.float16, device="cuda")
    v = torch.empty_like(k)
    dp.qkv_project(h.cuda(), wts["w_qkv"].cuda(), wts["b_qkv"].cuda(), q, k, v)
    dp.device_status()
    exact = O.linear(h, wts["w_qkv"], wts["b_qkv"])
    dot = _dot_bound(O.as_f64(h), O.as_f64(wts["w_qkv"]))
    for got, sl, unit in ((q, slice(0, D), 2.0 ** -8), (k, slice(D, 2 * D), 2.0 ** -11),
                          (v, slice(2 * D, 3 * D), 2.0 ** -11)):
        e = exact[:, sl]
        assert np.all(np.abs(got.cpu().double().numpy() - e) <= unit * np.abs(e) + dot[:, sl] + 1e-7)


def test_qkv_project_saturates_k_v_at_the_f16_limit(dp):
    """k and v leave the projection as f16 features: a value beyond f16's range stores as
    +-65504 (saturating, not inf).  Large weights push whole columns of k and v past the
    limit, both signs; q (bf16) keeps the exact value to one bf16 unit."""
    D, m = 256, 130
    h = torch.full((m, D), 2.0, dtype=torch.bfloat16)
    w = torch.zeros(3 * D, D)
    w[:D] = 0.01
    w[D:D + 8] = 200.0            # k columns 0..7: 256 * 2 * 200 = 102400
    w[2 * D:2 * D + 8] = -150.0   # v columns 0..7: -76800
    w[D + 8:D + 16] = 100.0       # k columns 8..15: 51200, in range
    w = w.to(torch.bfloat16)
    q = torch.empty(m, D, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(m, D, dtype=torch.float16, device="cuda")
    v = torch.empty_like(k)
    dp.qkv_project(h.cuda(), w.cuda(), None, q, k, v)
    dp.device_status()
    exact = O.linear(h, w, None)
    kg, vg = k.cpu().double().numpy(), v.cpu().double().numpy()
    assert np.all(np.isfinite(kg)) and np.all(np.isfinite(vg))
    assert np.all(kg[:, :8] == 65504.0) and np.all(vg[:, :8] == -65504.0)
    assert np.all(np.abs(kg[:, 8:16] - exact[:, D + 8:D + 16]) <= 2.0 ** -11 * np.abs(exact[:, D + 8:D + 16]))
    assert np.all(np.abs(q.cpu().double().numpy() - exact[:, :D]) <= 2.0 ** -8 * np.abs(exact[:, :D]) + 1e-6)
    assert np.array_equal(kg, O.round_to(exact[:, D:2 * D], "f16"))


def test_out_project_gated_residual(dp):
    D, rows = 768, [100, 156, 44]
    m = sum(rows)
    o, x = _bf16((m, D), 8), _bf16((m, D), 9)
    wts = make_sublayer_weights(D, 10)
    table = _table(D, 11)
    ts = [3, 400, 998]
    blk = dp.blocks_from_table(table.cuda(), ts, rows)
    out = torch.empty(m, D, dtype=torch.bfloat16, device="cuda")
    dp.out_project(o.cuda(), wts["w_o"].cuda(), wts["b_o"].cuda(), blk, x.cuda(), out)
    dp.device_status()
    mod = O.lookup(table, ts)
    beta = O.row_blocks(np.cumsum([0] + rows), m)
    gate = mod[beta, 2, :]
    exact = O.as_f64(x) + gate * O.linear(o, wts["w_o"], wts["b_o"])
    bound = 2.0 ** -8 * np.abs(exact) + np.abs(gate) * _dot_bound(O.as_f64(o), O.as_f64(wts["w_o"])) + 1e-6
    assert np.all(np.abs(out.cpu().double().numpy() - exact) <= bound)


def _small_case(H, hd, rows, cache_len, seed):
    D = H * hd
    n = sum(rows)
    x = _bf16((n, D), seed)
    ck = _bf16((max(rows), D), seed + 1).to(torch.float16)
    cv = _bf16((max(rows), D), seed + 2).to(torch.float16)
    table = _table(D, seed + 3)
    ts = [int(t) for t in np.linspace(0, 999, len(rows)).round()]
    wts = make_sublayer_weights(D, seed + 4)
    return D, n, x, ck, cv, table, ts, wts


@pytest.mark.parametrize("H,hd,rows,cache_len", [(4, 64, [300, 300, 211], 200), (2, 128, [256, 129], 0),
                                                 (8, 64, [1000, 1000, 777], 1000)])
def test_sublayer_step_matches_oracle(dp, H, hd, rows, cache_len):
    D, n, x, ck, cv, table, ts, wts = _small_case(H, hd, rows, cache_len, 20 + H)
    cap = max(rows)
    blk = dp.blocks_from_table(table.cuda(), ts, rows)
    cache = dp.KVCache(cap, D, torch.float16, k=ck.cuda().view(1, cap, D).clone(),
                       v=cv.cuda().view(1, cap, D).clone(), length=cache_len)
    work = dp.sublayer_work(n, D)
    out = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
    w = {key: t.cuda() for key, t in wts.items()}
    dp.sublayer_step(x.cuda(), blk, w["w_qkv"], w["b_qkv"], w["w_o"], w["b_o"], cache, work, out, H, hd, EPS,
                     pop=True)
    dp.device_status()
    ro = list(np.cumsum([0] + rows))
    mod = O.lookup(table, ts)
    want, wk, wv = O.sublayer_step(x, wts["w_qkv"], wts["b_qkv"], wts["w_o"], wts["b_o"], ck, cv, cache_len, ro,
                                   mod, H, hd, EPS, rounded=True)
    assert_close(out.cpu().double().numpy(), want, "bf16", "sublayer step")
    plain, _, _ = O.sublayer_step(x, wts["w_qkv"], wts["b_qkv"], wts["w_o"], wts["b_o"], ck, cv, cache_len, ro,
                                  mod, H, hd, EPS, rounded=False)
    assert_close(out.cpu().double().numpy(), plain, "bf16", "sublayer step vs the plain definition")
    _, q_g, k_g, v_g = dp.sublayer_planes(work, n, D)
    # projected k, v: the GPU's fp32 pre-norm and the oracle's float64 one can round an h
    # element to neighbouring bf16 values (at most one unit, 2^-7 |h|, apart); through W that
    # moves k and v by at most 2^-7 sum_c |h_c| |w_c|, plus the f16 unit and the fp32 sum
    h = O.round_to(O.ln_modulate(x, ro, mod, EPS), "bf16")
    wabs = np.abs(O.as_f64(wts["w_qkv"]))
    for got, ref, sl in ((k_g, wk, slice(D, 2 * D)), (v_g, wv, slice(2 * D, 3 * D))):
        g = got.cpu().double().numpy()
        prop = np.abs(h) @ wabs[sl].T
        assert np.all(np.abs(g - ref) <= 2.0 ** -10 * np.abs(ref) + (2.0 ** -7 + 2.0 ** -12) * prop)
        assert np.mean(g == ref) > 0.95
    # the advance: the head block's projected k, v rows became the cache, bit for bit
    n0 = rows[0]
    assert cache.length == n0 and cache.n_advances == 1
    assert bytes_equal(cache.k[0, :n0], k_g[:n0]) and bytes_equal(cache.v[0, :n0], v_g[:n0])


def test_sublayer_step_second_step_uses_the_cache(dp):
    H, hd, rows = 4, 64, [200, 200]
    D, n, x, ck, cv, table, ts, wts = _small_case(H, hd, rows, 0, 40)
    blk = dp.blocks_from_table(table.cuda(), ts, rows)
    cache = dp.KVCache(200, D, torch.float16)
    work = dp.sublayer_work(n, D)
    out1 = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
    out2 = torch.empty_like(out1)
    w = {key: t.cuda() for key, t in wts.items()}
    xc = x.cuda()
    dp.sublayer_step(xc, blk, w["w_qkv"], w["b_qkv"], w["w_o"], w["b_o"], cache, work, out1, H, hd, pop=True)
    dp.sublayer_step(xc, blk, w["w_qkv"], w["b_qkv"], w["w_o"], w["b_o"], cache, work, out2, H, hd)
    dp.device_status()
    ro = [0, 200, 400]
    mod = O.lookup(table, ts)
    # second step: the cache holds the first step's head-block k, v (read back from the GPU)
    _, _, k_g, v_g = dp.sublayer_planes(work, n, D)
    want2, _, _ = O.sublayer_step(x, wts["w_qkv"], wts["b_qkv"], wts["w_o"], wts["b_o"], cache.k[0].cpu(),
                                  cache.v[0].cpu(), 200, ro, mod, H, hd, EPS, rounded=True)
    assert_close(out2.cpu().double().numpy(), want2, "bf16", "second step")
    plain2, _, _ = O.sublayer_step(x, wts["w_qkv"], wts["b_qkv"], wts["w_o"], wts["b_o"], cache.k[0].cpu(),
                                   cache.v[0].cpu(), 200, ro, mod, H, hd, EPS, rounded=False)
    assert_close(out2.cpu().double().numpy(), plain2, "bf16", "second step vs the plain definition")
    assert errors(out2.cpu().double().numpy(), out1.cpu().double().numpy())[0] > 1e-3


def test_sublayer_step_full_size_sampled(dp):
    """CogVideo-like window (4 x 2700 rows, 2700-row cache, 48 x 64 heads) in the launch
    configuration the benchmark times; the oracle computes the projections for all rows
    and the attention and output for sampled rows."""
    cfg = step_config("cogvideo_bf16")
    x_in = make_step_inputs(cfg)
    H, hd, D, n = cfg.n_heads, cfg.head_dim, cfg.hidden, cfg.n_win
    x = (x_in["q"].float() * 8.0).to(torch.bfloat16)       # the window's hidden state, N(0, 1)
    wts = make_sublayer_weights(D, cfg.seed + 100)
    ck, cv = as_features(x_in["cache_k"], cfg.dtype), as_features(x_in["cache_v"], cfg.dtype)
    blk = dp.blocks_from_table(x_in["table"].cuda(), x_in["timesteps"], cfg.block_rows)
    cache = dp.KVCache(cfg.cache_capacity, D, torch.float16, k=ck.cuda().view(1, -1, D).clone(),
                       v=cv.cuda().view(1, -1, D).clone(), length=cfg.cache_len)
    work = dp.sublayer_work(n, D)
    out = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
    w = {key: t.cuda() for key, t in wts.items()}
    dp.sublayer_step(x.cuda(), blk, w["w_qkv"], w["b_qkv"], w["w_o"], w["b_o"], cache, work, out, H, hd, EPS,
                     pop=True)
    dp.device_status()
    rows = sample_rows(cfg.row_offset, n_extra=48)
    mod = O.lookup(x_in["table"], x_in["timesteps"])
    want, _, _ = O.sublayer_step(x, wts["w_qkv"], wts["b_qkv"], wts["w_o"], wts["b_o"], ck, cv, cfg.cache_len,
                                 cfg.row_offset, mod, H, hd, EPS, rounded=True, rows=rows)
    assert_close(out[rows].cpu().double().numpy(), want, "bf16", "cogvideo sublayer")
    plain, _, _ = O.sublayer_step(x, wts["w_qkv"], wts["b_qkv"], wts["w_o"], wts["b_o"], ck, cv, cfg.cache_len,
                                  cfg.row_offset, mod, H, hd, EPS, rounded=False, rows=rows)
    assert_close(out[rows].cpu().double().numpy(), plain, "bf16", "cogvideo sublayer vs the plain definition")
    _, _, k_g, v_g = dp.sublayer_planes(work, n, D)
    n0 = cfg.block_rows[0]
    assert bytes_equal(cache.k[0, :n0], k_g[:n0]) and bytes_equal(cache.v[0, :n0], v_g[:n0])

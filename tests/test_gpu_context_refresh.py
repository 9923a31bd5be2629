"""GPU parity of the fresh-context variant of the feature cache (the context block's K/V
recomputed at the step that uses them instead of reused from its last evaluation) against
the float64 oracle, through the C ABI.

Recomputed from the same rows with the same conditioning, the features must equal, bit for
bit, what the cached variant stored (the same kernels compute both); recomputed with other
conditioning they follow the oracle's definition, and a step that attends to them matches
the oracle's step over the recomputed context."""
import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import assert_close, bytes_equal
from workloads import make_sublayer_weights

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

EPS = 1e-6


def _table(D, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.tanh(torch.randn(1000, 3, D, generator=g))


def _rows(shape, seed, std=1.0, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * std).to(dtype)


# ----------------------------------------------------------------------------- sublayer

def _sublayer_case(H, hd, rows, seed):
    D = H * hd
    n = sum(rows)
    x = _rows((n, D), seed)
    table = _table(D, seed + 1)
    ts = [int(t) for t in np.linspace(0, 999, len(rows)).round()]
    wts = make_sublayer_weights(D, seed + 2)
    return D, n, x, table, ts, wts


@pytest.mark.parametrize("H,hd,rows", [(4, 64, [300, 300, 211]), (2, 128, [129, 256]), (8, 64, [1000, 77])])
def test_sublayer_refresh_equals_cached_features(dp, H, hd, rows):
    """Context recomputed from the exited block's rows and conditioning == what the cached
    variant's advance stored, bit for bit; a later block's rows, recomputed alone, equal
    that block's rows of the step's own k, v planes."""
    D, n, x, table, ts, wts = _sublayer_case(H, hd, rows, 50 + H)
    cap = max(rows)
    w = {key: t.cuda() for key, t in wts.items()}
    xc = x.cuda()
    tab = table.cuda()
    blk = dp.blocks_from_table(tab, ts, rows)
    cached = dp.KVCache(cap, D, torch.float16)
    work = dp.sublayer_work(n, D)
    out = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
    dp.sublayer_step(xc, blk, w["w_qkv"], w["b_qkv"], w["w_o"], w["b_o"], cached, work, out, H, hd, EPS, pop=True)
    _, _, k_g, v_g = dp.sublayer_planes(work, n, D)
    k_g, v_g = k_g.clone(), v_g.clone()
    n0 = rows[0]
    fresh = dp.KVCache(cap, D, torch.float16)
    scratch = torch.empty(cap * D, dtype=torch.bfloat16, device="cuda")
    dp.context_refresh_sublayer(xc[:n0], dp.blocks_from_table(tab, ts[:1], [n0]), w["w_qkv"], w["b_qkv"], fresh,
                                scratch, EPS)
    dp.device_status()
    assert fresh.length == n0 and fresh.n_advances == 0
    assert bytes_equal(fresh.k[0, :n0], cached.k[0, :n0]) and bytes_equal(fresh.v[0, :n0], cached.v[0, :n0])
    r0, r1 = rows[0], rows[0] + rows[1]
    dp.context_refresh_sublayer(xc[r0:r1], dp.blocks_from_table(tab, ts[1:2], [r1 - r0]), w["w_qkv"], w["b_qkv"],
                                fresh, scratch, EPS)
    dp.device_status()
    assert fresh.length == r1 - r0
    assert bytes_equal(fresh.k[0, :r1 - r0], k_g[r0:r1]) and bytes_equal(fresh.v[0, :r1 - r0], v_g[r0:r1])


@pytest.mark.parametrize("H,hd,n_ctx,t_ctx", [(4, 64, 300, 0), (2, 128, 129, 500), (8, 64, 1, 999)])
def test_sublayer_fresh_step_matches_oracle(dp, H, hd, n_ctx, t_ctx):
    """Refresh the context (its own rows, conditioned on timestep t_ctx), then a step with no
    advance: features and output against the oracle's fresh context and step."""
    rows = [256, 200, 57]
    D, n, x, table, ts, wts = _sublayer_case(H, hd, rows, 70 + n_ctx)
    x_ctx = _rows((n_ctx, D), 90 + n_ctx)
    w = {key: t.cuda() for key, t in wts.items()}
    tab = table.cuda()
    cache = dp.KVCache(512, D, torch.float16, length=0)
    cache.k.fill_(7.0)
    cache.v.fill_(7.0)
    work = dp.sublayer_work(n, D)
    dp.context_refresh_sublayer(x_ctx.cuda(), dp.blocks_from_table(tab, [t_ctx], [n_ctx]), w["w_qkv"], w["b_qkv"],
                                cache, work, EPS)
    out = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
    dp.sublayer_step(x.cuda(), dp.blocks_from_table(tab, ts, rows), w["w_qkv"], w["b_qkv"], w["w_o"], w["b_o"],
                     cache, work, out, H, hd, EPS)
    dp.device_status()
    assert cache.length == n_ctx and cache.n_advances == 0
    mod_ctx = O.lookup(table, [t_ctx])
    fk, fv = O.fresh_context_sublayer(x_ctx, [0, n_ctx], mod_ctx, wts["w_qkv"], wts["b_qkv"], EPS, rounded=True)
    # features: one bf16 unit of h (2^-7 |h|) through W, the f16 unit and the fp32 sum
    h = O.round_to(O.ln_modulate(x_ctx, [0, n_ctx], mod_ctx, EPS), "bf16")
    wabs = np.abs(O.as_f64(wts["w_qkv"]))
    for got, ref, sl in ((cache.k[0, :n_ctx], fk, slice(D, 2 * D)), (cache.v[0, :n_ctx], fv, slice(2 * D, 3 * D))):
        g = got.cpu().double().numpy()
        prop = np.abs(h) @ wabs[sl].T
        assert np.all(np.abs(g - ref) <= 2.0 ** -10 * np.abs(ref) + (2.0 ** -7 + 2.0 ** -12) * prop)
        assert np.mean(g == ref) > 0.95
    # rows beyond the context keep whatever the slot held (not read: len = n_ctx)
    assert bool((cache.k[0, n_ctx:] == 7.0).all())
    want, _, _ = O.sublayer_step(x, wts["w_qkv"], wts["b_qkv"], wts["w_o"], wts["b_o"], fk, fv, n_ctx,
                                 list(np.cumsum([0] + rows)), O.lookup(table, ts), H, hd, EPS, rounded=True)
    assert_close(out.cpu().double().numpy(), want, "bf16", "step over the fresh context")
    # and against the plain definition: the context's features and the step, nothing rounded
    pk, pv = O.fresh_context_sublayer(x_ctx, [0, n_ctx], mod_ctx, wts["w_qkv"], wts["b_qkv"], EPS, rounded=False)
    plain, _, _ = O.sublayer_step(x, wts["w_qkv"], wts["b_qkv"], wts["w_o"], wts["b_o"], pk, pv, n_ctx,
                                  list(np.cumsum([0] + rows)), O.lookup(table, ts), H, hd, EPS, rounded=False)
    assert_close(out.cpu().double().numpy(), plain, "bf16", "step over the fresh context vs the plain definition")


# ----------------------------------------------------------------------------- window step

@pytest.mark.parametrize("dtype,H,hd,rows", [("bf16", 4, 64, [300, 211]), ("f32", 2, 64, [128, 128]),
                                             ("bf16", 2, 128, [129, 1])])
def test_identity_refresh_equals_cached_and_oracle(dp, dtype, H, hd, rows):
    """Window-step features: recomputed from the exited block's k, v rows == the advance's
    copy bit for bit, and == the oracle's rounding of the definition; a step over a context
    recomputed at another timestep matches the oracle's step."""
    D = H * hd
    n = sum(rows)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    fdt = dp.feature_dtype(tdt)
    q, k, v = (_rows((n, D), 110 + i, 0.5, tdt) for i in range(3))
    table = _table(D, 113)
    tab = table.cuda()
    ts = [0, 999][:len(rows)]
    blk = dp.blocks_from_table(tab, ts, rows)
    cap = max(rows)
    cached = dp.KVCache(cap, D, fdt)
    kv_work = torch.empty(2, n, D, dtype=fdt, device="cuda")
    out = torch.empty(n, D, dtype=tdt, device="cuda")
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    dp.window_step(qc, kc, vc, blk, cached, kv_work, out, H, hd, pop=True)
    n0 = rows[0]
    fresh = dp.KVCache(cap, D, fdt)
    dp.context_refresh(kc[:n0], vc[:n0], dp.blocks_from_table(tab, ts[:1], [n0]), fresh)
    dp.device_status()
    assert fresh.length == n0
    assert bytes_equal(fresh.k[0, :n0], cached.k[0, :n0]) and bytes_equal(fresh.v[0, :n0], cached.v[0, :n0])
    # conditioned on another timestep: the oracle's rounding of the definition, bit for bit
    t_ctx = 421
    mod_ctx = O.lookup(table, [t_ctx])
    dp.context_refresh(kc[:n0], vc[:n0], dp.blocks_from_table(tab, [t_ctx], [n0]), fresh)
    out2 = torch.empty_like(out)
    dp.window_step(qc, kc, vc, blk, fresh, kv_work, out2, H, hd)
    dp.device_status()
    rdt = "f16" if dtype == "bf16" else "f32"
    assert np.array_equal(fresh.k[0, :n0].cpu().double().numpy(), O.modulate_rounded(k[:n0], [0, n0], mod_ctx, rdt))
    assert np.array_equal(fresh.v[0, :n0].cpu().double().numpy(), O.modulate_rounded(v[:n0], [0, n0], mod_ctx, rdt))
    fk, fv = O.fresh_context(k[:n0], v[:n0], [0, n0], mod_ctx)
    want, _, _ = O.window_step(q, k, v, fk, fv, n0, list(np.cumsum([0] + rows)), O.lookup(table, ts), H, hd)
    assert_close(out2.cpu().double().numpy(), want, dtype, "window step over the fresh context")


def test_refresh_writes_only_the_slot_attention_reads(dp):
    """Cache ring of 3 slots after 4 advances: the refresh overwrites slot (4 - 1) mod 3 = 0
    only; with every slot read, the step sees the older slots' cached rows and the fresh
    ones."""
    H, hd = 4, 64
    D = H * hd
    rows = [128, 100]
    n = sum(rows)
    table = _table(D, 120)
    tab = table.cuda()
    cache = dp.KVCache(128, D, torch.float16, n_slots=3)
    kv_work = torch.empty(2, n, D, dtype=torch.float16, device="cuda")
    out = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
    blk = dp.blocks_from_table(tab, [0, 999], rows)
    for s in range(4):
        q, k, v = (_rows((n, D), 130 + 3 * s + i, 0.5).cuda() for i in range(3))
        dp.window_step(q, k, v, blk, cache, kv_work, out, H, hd, pop=True)
    dp.device_status()
    assert cache.read_slot() == 0
    before = (cache.k.clone(), cache.v.clone(), [cache.desc.len[i] for i in range(3)])
    x_ctx = _rows((77, D), 150, 0.5).cuda()
    dp.context_refresh(x_ctx, x_ctx, dp.blocks_from_table(tab, [0], [77]), cache)
    out_all = torch.empty_like(out)
    dp.window_step(q, k, v, blk, cache, kv_work, out_all, H, hd, cache_all_slots=True)
    dp.device_status()
    assert [cache.desc.len[i] for i in range(3)] == [77] + before[2][1:]
    assert bytes_equal(cache.k[1:], before[0][1:]) and bytes_equal(cache.v[1:], before[1][1:])
    assert bytes_equal(cache.k[0, 77:], before[0][0, 77:])
    # oracle: the slots oldest first (1, 2, then the refreshed 0), then the window
    ck = torch.cat([cache.k[1, :before[2][1]], cache.k[2, :before[2][2]], cache.k[0, :77]]).cpu()
    cv = torch.cat([cache.v[1, :before[2][1]], cache.v[2, :before[2][2]], cache.v[0, :77]]).cpu()
    mod = O.lookup(table, [0, 999])
    want, _, _ = O.window_step(q.cpu(), k.cpu(), v.cpu(), ck, cv, ck.shape[0], [0, 128, n], mod, H, hd)
    assert_close(out_all.cpu().double().numpy(), want, "bf16", "every slot, slot 0 refreshed")


# ----------------------------------------------------------------------------- the long run

def _long_run_sums(dp, fresh_t, max_steps=None):
    """Per-step checksums of the long run's outputs (int64 sums of the bf16 bit patterns)."""
    from workloads import make_run_noise, make_run_table, run_config
    rc = run_config()
    H, hd, D, W, T = rc.n_heads, rc.head_dim, rc.hidden, rc.window_blocks, rc.n_timesteps
    noise = [b.cuda() for b in make_run_noise(rc)]
    table = make_run_table(rc).cuda()
    tau = O.timestep_schedule(T)
    cache = dp.KVCache(rc.slot_rows, D, torch.float16)
    queue = dp.Queue(W + 1, rc.slot_rows, D)
    n_max = W * rc.slot_rows
    kv = torch.empty(2 * n_max * D, dtype=torch.float16, device="cuda")
    out = torch.empty(n_max, D, dtype=torch.bfloat16, device="cuda")
    sums, pops = [], []

    def on_step(step, n, popped, pushed):
        sums.append(out[:n].view(torch.int16).sum(dtype=torch.int64))
        pops.append(popped)

    steps = dp.run_fifo(noise, table, tau, W, cache, queue, kv, out, H, hd, on_step=on_step, max_steps=max_steps,
                        fresh_t=fresh_t)
    dp.device_status()
    return torch.stack(sums).cpu(), pops, steps


def test_long_run_fresh_context_at_the_final_timestep_equals_cached(dp):
    """The whole run with the context recomputed before every step from the exited block's
    latent rows at timestep 0 (where its last evaluation ran) gives the cached run's outputs
    bit for bit at every one of the 850 steps; conditioned on another timestep it does not."""
    cached, pops, n = _long_run_sums(dp, None)
    fresh, pops_f, n_f = _long_run_sums(dp, 0)
    assert n == n_f == 850 and pops == pops_f
    assert torch.equal(cached, fresh)
    first_exit = pops.index(True)
    other, _, _ = _long_run_sums(dp, 500, max_steps=first_exit + 3)
    assert torch.equal(other[:first_exit + 1], cached[:first_exit + 1])   # no context yet, or the same one
    assert not torch.equal(other[first_exit + 1:], cached[first_exit + 1:first_exit + 3])
    with pytest.raises(ValueError):
        from workloads import run_config
        rc = run_config()
        q = dp.Queue(rc.window_blocks, rc.slot_rows, rc.hidden)
        dp.run_fifo([], torch.zeros(1000, 3, rc.hidden, device="cuda"), [0], rc.window_blocks,
                    dp.KVCache(rc.slot_rows, rc.hidden, torch.float16), q, None, None, 1, 1, fresh_t=0)

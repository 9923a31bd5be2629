"""GPU parity: every kernel of the window step against the CPU oracle on seeded inputs,
through the C ABI (the Python binding marshals arguments only)."""
import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import assert_close, bytes_equal, errors, sample_rows
from workloads import as_features, make_step_inputs, step_config, to_dtype

TDT = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _table(D, seed=5, T=1000):
    g = torch.Generator().manual_seed(seed)
    return torch.tanh(torch.randn(T, 3, D, generator=g)).contiguous()


def _randn(shape, seed, dtype, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return to_dtype(torch.randn(*shape, generator=g) * std, dtype)


# --------------------------------------------------------------------------- A1 modulation

@pytest.mark.parametrize("dtypes", [("bf16", "f16"), ("bf16", "bf16"), ("f32", "f32")])
@pytest.mark.parametrize("rows", [[300, 450, 250], [1], [0, 7, 129, 0]])
def test_modulate_matches_oracle_bitwise(dp, dtypes, rows):
    x_dt, dtype = dtypes
    D = 1536
    n = sum(rows)
    x = _randn((n, D), 1, x_dt)
    table = _table(D)
    ts = [int(t) for t in np.linspace(0, 999, len(rows)).round()]
    xd, td = x.cuda(), table.cuda()
    y = torch.empty(n, D, dtype=TDT[dtype], device="cuda")
    blk = dp.blocks_from_table(td, ts, rows)
    dp.adaln_modulate(xd, y, blk)
    ro = blk.offsets
    mod = O.lookup(table, ts)
    want = O.modulate_rounded(x, ro, mod, dtype)
    got = y.cpu().double().numpy()
    assert np.array_equal(got, want), f"mismatches: {int((got != want).sum())}"
    # against the float64 definition: one rounding to the storage type (unit roundoff u,
    # plus half the smallest subnormal eta/2 for gradual underflow) and the fp32 rounding of
    # 1 + scale, which matters where x * (1 + scale) and shift nearly cancel
    exact = O.modulate(x, ro, mod)
    beta = O.row_blocks(ro, n)
    xf = O.as_f64(x)
    u = {"bf16": 2.0 ** -8, "f16": 2.0 ** -11, "f32": 2.0 ** -24}[dtype]
    half_eta = {"bf16": 2.0 ** -134, "f16": 2.0 ** -25, "f32": 2.0 ** -150}[dtype]
    bound = (u * np.abs(exact) + half_eta +
             2.0 ** -22 * (np.abs(xf * (1.0 + mod[beta, 1])) + np.abs(mod[beta, 0])))
    assert np.all(np.abs(got - exact) <= bound)
    if x_dt == dtype:                       # in place gives the same bytes
        dp.adaln_modulate(xd, xd, blk)
        assert bytes_equal(xd, y)


# --------------------------------------------------------------------------- A2 attention

ATTN_CASES = [
    # (H, hd, block rows, cache_len, cache capacity, residual, flags, feature dtype)
    (2, 64, [500, 300, 200], 300, 333, False, 3, "f16"),
    (2, 128, [400, 377], 0, 16, True, 3, "f16"),
    (3, 64, [129], 1, 8, False, 3, "f16"),
    (1, 64, [1], 0, 1, False, 3, "f16"),
    (2, 128, [256, 256], 128, 128, True, 0, "f16"),
    (4, 64, [100, 0, 156, 1], 200, 256, True, 1, "f16"),
    (2, 64, [5000], 2500, 2500, False, 2, "f16"),
    (2, 64, [700, 300], 300, 300, False, 3, "bf16"),
    (2, 128, [257, 255], 100, 100, True, 3, "bf16"),
]


@pytest.mark.parametrize("case", ATTN_CASES, ids=lambda c: f"H{c[0]}_hd{c[1]}_n{sum(c[2])}_c{c[3]}_{c[7]}")
def test_attention_bf16_matches_oracle(dp, case):
    H, hd, rows, Lc, cap, with_res, flags, ft = case
    D = H * hd
    n = sum(rows)
    q = _randn((n, D), 11, "bf16")
    k, v = (_randn((n, D), s, "bf16").to(TDT[ft]) for s in (12, 13))
    ck, cv = (_randn((cap, D), s, "bf16").to(TDT[ft]) for s in (14, 15))
    res = _randn((n, D), 16, "bf16") if with_res else None
    table = _table(D)
    ts = [int(t) for t in np.linspace(0, 999, len(rows)).round()]
    blk = dp.blocks_from_table(table.cuda(), ts, rows)
    out = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
    dp.window_attention(q.cuda(), k.cuda(), v.cuda(), ck.cuda(), cv.cuda(), Lc, out, H, hd, blk, flags=flags,
                        residual=res.cuda() if res is not None else None)
    dp.device_status()
    want = O.window_attention(q, k, v, ck, cv, Lc, blk.offsets, O.lookup(table, ts), H, hd,
                              mod_q=bool(flags & 1), gate_out=bool(flags & 2), residual=res)
    assert_close(out.cpu().double().numpy(), want, "bf16", f"attention {case}")


def _jump_case(hd, cache_len, n_win, seed=31, levels=None):
    """Queries in groups of 128 rows, each group with its own direction (dim g of every head);
    keys planted on that direction at chosen logit levels (log2 units: x = q.k * scale *
    log2(e)), so that the running reference max of the softmax jumps by more than 2^8 in
    chosen 32-key chunks of chosen key tiles, with groups of keys just below each jump
    carrying a visible share of the row's weight.  Key index = position in [cache ; window]."""
    BN = 128 if hd == 64 else 64
    nch = BN // 32
    key = lambda t, i, o: t * BN + 32 * min(i, nch - 1) + o
    plan = levels(key, nch) if levels else {   # every group on tiles of its own
        0: [(key(1, c, o), 3.0) for c in range(nch - 1) for o in range(32)] + [(key(1, nch - 1, 5), 11.5)],
        1: [(key(2, 0, o), 3.0) for o in range(31) if o != 7] + [(key(2, 0, 7), 11.6)],
        2: [(key(3, 1, 3), 9.0), (key(6, nch - 2, 10), 18.0)],
        3: [(key(4, 0, o), 2.0) for o in range(1, 32)] + [(key(4, 0, 0), 9.0), (key(4, nch - 1, 31), 18.2)],
    }
    assert len({j for keys in plan.values() for j, _ in keys}) == sum(len(keys) for keys in plan.values())
    H = 2
    D = H * hd
    g = torch.Generator().manual_seed(seed)
    L = cache_len + n_win
    q = torch.randn(n_win, D, generator=g) * 0.5
    kall = torch.randn(L, D, generator=g) * 0.05
    vall = torch.randn(L, D, generator=g)
    a, s = 4.0, hd ** -0.5
    for h in range(H):
        q[:, h * hd:h * hd + 4] = 0.0
        for grp, keys in plan.items():
            rows = slice(128 * grp, 128 * (grp + 1))
            q[rows, h * hd + grp] = a
            for j, x in keys:
                kall[j, h * hd:h * hd + 4] = 0.0
                kall[j, h * hd + grp] = x / (a * s * 1.4426950408889634)
    q = q.to(torch.bfloat16)
    kall, vall = kall.to(torch.float16), vall.to(torch.float16)
    return H, D, q, kall[cache_len:].contiguous(), vall[cache_len:].contiguous(), kall[:cache_len].contiguous(), \
        vall[:cache_len].contiguous()


@pytest.mark.parametrize("hd,cache_len", [(64, 0), (64, 168), (128, 0), (128, 100)])
def test_attention_reference_max_jumps_mid_tile(dp, hd, cache_len):
    """The softmax's reference max moves by more than 2^8 inside a key tile (in its first,
    middle and last 32-key chunk, twice in one tile, over a ragged cache-window boundary):
    O, the row sum and the P chunks already computed are rescaled."""
    n = 1024
    H, D, q, k, v, ck, cv = _jump_case(hd, cache_len, n)
    cap = max(cache_len, 1)
    ckd = ck.cuda() if cache_len else torch.zeros(cap, D, dtype=torch.float16, device="cuda")
    cvd = cv.cuda() if cache_len else torch.zeros(cap, D, dtype=torch.float16, device="cuda")
    table = _table(D)
    blk = dp.blocks_from_table(table.cuda(), [0], [n])
    out = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
    dp.window_attention(q.cuda(), k.cuda(), v.cuda(), ckd, cvd, cache_len, out, H, hd, blk, flags=0)
    dp.device_status()
    want = O.window_attention(q, k, v, ck if cache_len else ckd.cpu(), cv if cache_len else cvd.cpu(), cache_len,
                              blk.offsets, O.lookup(table, [0]), H, hd, mod_q=False, gate_out=False)
    assert_close(out.cpu().double().numpy(), want, "bf16", f"max jumps hd {hd} cache {cache_len}")
    # the planted keys decide the result: each group's output is far from the mean of V
    assert np.abs(want[:512]).max() > 0.5


# Jumps past the range of fp32 exp2 (2^x is infinite from x = 128 on): single keys 60 to 400
# log2 units above everything before them, in columns of either exp2 unit (column 0 of a
# 32-key chunk and its last column; column 7), some in the same tile as a smaller jump.
def _far_levels(key, nch):
    return {
        0: [(key(1, 0, 0), 150.0)],
        1: [(key(2, 0, o), 3.0) for o in range(8, 31)] + [(key(2, 0, 7), 200.0)],
        2: [(key(3, nch - 1, 3), 60.0), (key(6, 0, 10), 300.0)],
        3: [(key(4, 0, 0), 130.0), (key(4, nch - 1, 31), 400.0)],
    }


@pytest.mark.parametrize("hd,cache_len", [(64, 0), (64, 168), (128, 0), (128, 100)])
def test_attention_reference_max_jumps_past_fp32_exp2_range(dp, hd, cache_len):
    """Scores that jump by 60 to 400 log2 units within the row: each row's output is, to
    within the tolerance, the value row of its largest key, whatever came before it."""
    n = 1024
    H, D, q, k, v, ck, cv = _jump_case(hd, cache_len, n, seed=37, levels=_far_levels)
    cap = max(cache_len, 1)
    ckd = ck.cuda() if cache_len else torch.zeros(cap, D, dtype=torch.float16, device="cuda")
    cvd = cv.cuda() if cache_len else torch.zeros(cap, D, dtype=torch.float16, device="cuda")
    table = _table(D)
    blk = dp.blocks_from_table(table.cuda(), [0], [n])
    out = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
    dp.window_attention(q.cuda(), k.cuda(), v.cuda(), ckd, cvd, cache_len, out, H, hd, blk, flags=0)
    dp.device_status()
    want = O.window_attention(q, k, v, ck if cache_len else ckd.cpu(), cv if cache_len else cvd.cpu(), cache_len,
                              blk.offsets, O.lookup(table, [0]), H, hd, mod_q=False, gate_out=False)
    got = out.cpu().double().numpy()
    assert np.isfinite(got).all()
    assert_close(got, want, "bf16", f"far jumps hd {hd} cache {cache_len}")
    # one key holds all the weight: the first 512 rows equal a value row of V
    assert np.abs(want[:512]).max() > 0.5


def test_attention_bf16_deterministic(dp):
    H, hd, n, Lc = 4, 64, 1000, 300
    D = H * hd
    q = _randn((n, D), 0, "bf16").cuda()
    k, v, ck, cv = (_randn((n, D), s, "bf16").to(torch.float16).cuda() for s in range(1, 5))
    blk = dp.blocks_from_table(_table(D).cuda(), [0, 500], [600, 400])
    a = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
    b = torch.empty_like(a)
    dp.window_attention(q, k, v, ck, cv, Lc, a, H, hd, blk)
    dp.window_attention(q, k, v, ck, cv, Lc, b, H, hd, blk)
    assert bytes_equal(a, b)


@pytest.mark.parametrize("hd", [64, 16])
def test_attention_f32_matches_oracle(dp, hd):
    H = 2
    D = H * hd
    rows = [100, 90]
    n = sum(rows)
    q, k, v = (_randn((n, D), s, "f32") for s in (21, 22, 23))
    ck, cv = (_randn((70, D), s, "f32") for s in (24, 25))
    res = _randn((n, D), 26, "f32")
    table = _table(D)
    blk = dp.blocks_from_table(table.cuda(), [500, 999], rows)
    out = torch.empty(n, D, dtype=torch.float32, device="cuda")
    dp.window_attention(q.cuda(), k.cuda(), v.cuda(), ck.cuda(), cv.cuda(), 70, out, H, hd, blk,
                        residual=res.cuda())
    want = O.window_attention(q, k, v, ck, cv, 70, blk.offsets, O.lookup(table, [500, 999]), H, hd, residual=res)
    assert_close(out.cpu().double().numpy(), want, "f32", "f32 attention")


# --------------------------------------------------------------------------- A3 advance

def test_kvcache_advance_bitexact_ring(dp):
    D, cap = 256, 96
    c = dp.KVCache(cap, D, dtype=torch.bfloat16, n_slots=3)
    ref = O.KVCacheRing(3, cap, D)
    for a, n in enumerate([96, 50, 96, 1, 0, 96, 33]):
        ke, ve = _randn((max(n, 1), D), 100 + a, "bf16"), _randn((max(n, 1), D), 200 + a, "bf16")
        dp.kvcache_advance(c, ke.cuda(), ve.cuda(), n)
        slot = ref.advance(ke, ve, n)
        assert c.n_advances == a + 1 and c.read_slot() == slot and c.length == n
        torch.cuda.synchronize()
        assert np.array_equal(c.k[slot, :n].cpu().double().numpy(), ref.k[slot, :n])
        assert np.array_equal(c.v[slot, :n].cpu().double().numpy(), ref.v[slot, :n])
    with pytest.raises(dp.DpError):
        dp.kvcache_advance(c, ke.cuda(), ve.cuda(), cap + 1)


def test_queue_push_pop_mirrored_window(dp):
    D, slot = 128, 64
    qu = dp.Queue(3, slot, D, dtype=torch.bfloat16)
    ref = O.FifoQueue(3)
    blocks = [_randn((slot, D), 300 + i, "bf16") for i in range(7)] + [_randn((40, D), 399, "bf16")]
    pushed = 0
    for i, blk in enumerate(blocks):
        if qu.count == 3:
            dp.queue_pop(qu)
            ref.pop()
        dp.queue_push(qu, blk.cuda())
        ref.push(blk)
        pushed += 1
        torch.cuda.synchronize()
        assert qu.rows() == [b.latent.shape[0] for b in ref.blocks]
        assert np.array_equal(qu.window().cpu().double().numpy(), ref.window())
    with pytest.raises(dp.DpError):   # nothing may follow the short final block
        dp.queue_pop(qu)
        dp.queue_push(qu, blocks[0].cuda())


# --------------------------------------------------------------------------- A4 window step

def test_window_step_tiny_f32_two_steps(dp):
    """tiny_f32: one step with the preset cache, one advance, then a second step that must
    use the new cache (the exited head block's k')."""
    cfg = step_config("tiny_f32")
    x = make_step_inputs(cfg)
    H, hd, D, n = cfg.n_heads, cfg.head_dim, cfg.hidden, cfg.n_win
    table = x["table"].cuda()
    blk = dp.blocks_from_table(table, x["timesteps"], cfg.block_rows)
    ck = x["cache_k"].cuda().view(1, cfg.cache_capacity, D).clone()
    cv = x["cache_v"].cuda().view(1, cfg.cache_capacity, D).clone()
    cache = dp.KVCache(cfg.cache_capacity, D, torch.float32, k=ck, v=cv, length=cfg.cache_len)
    qu = dp.Queue(2, 128, D, dtype=torch.float32)
    for b in range(2):
        dp.queue_push(qu, x["noise"].cuda())
    q, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
    kv = torch.empty(2, n, D, dtype=torch.float32, device="cuda")
    out = torch.empty(n, D, dtype=torch.float32, device="cuda")
    dp.window_step(q, k, v, blk, cache, kv, out, H, hd, pop=True, queue=qu, push_noise=x["noise"].cuda())
    dp.device_status()
    mod = O.lookup(x["table"], x["timesteps"])
    want, kp, vp = O.window_step(x["q"], x["k"], x["v"], x["cache_k"], x["cache_v"], cfg.cache_len, cfg.row_offset,
                                 mod, H, hd)
    assert_close(out.cpu().double().numpy(), want, "f32", "step 1")
    # advance: the cache now holds the head block's k'/v' (bit-exact vs the rounded oracle)
    n0 = cfg.block_rows[0]
    kr = O.modulate_rounded(x["k"], cfg.row_offset, mod, "f32")
    vr = O.modulate_rounded(x["v"], cfg.row_offset, mod, "f32")
    assert cache.length == n0 and cache.n_advances == 1
    assert np.array_equal(cache.k[0, :n0].cpu().double().numpy(), kr[:n0])
    assert np.array_equal(cache.v[0, :n0].cpu().double().numpy(), vr[:n0])
    assert bytes_equal(cache.k[0, :n0], kv[0, :n0])
    assert qu.count == 2 and qu.evals() == [1, 0]
    # step 2 attends to the new cache
    out2 = torch.empty_like(out)
    dp.window_step(q, k, v, blk, cache, kv, out2, H, hd)
    want2, _, _ = O.window_step(x["q"], x["k"], x["v"], kr, vr, n0, cfg.row_offset, mod, H, hd)
    assert_close(out2.cpu().double().numpy(), want2, "f32", "step 2")
    assert errors(out2.cpu().double().numpy(), want)[0] > 1e-3   # the cache did change the result


@pytest.mark.parametrize("name", ["cogvideo_bf16", "wan_bf16", "longrun_steady_bf16", "wan_paper_bf16"])
def test_window_step_full_size_sampled(dp, name):
    """Full-size bf16 step in the launch configuration the benchmark times; the oracle
    computes sampled rows (block boundaries, first/last, ragged tail, random)."""
    cfg = step_config(name)
    x = make_step_inputs(cfg)
    H, hd, D, n = cfg.n_heads, cfg.head_dim, cfg.hidden, cfg.n_win
    blk = dp.blocks_from_table(x["table"].cuda(), x["timesteps"], cfg.block_rows)
    ck, cv = as_features(x["cache_k"], cfg.dtype), as_features(x["cache_v"], cfg.dtype)
    cache = dp.KVCache(cfg.cache_capacity, D, torch.float16, k=ck.cuda().view(1, -1, D),
                       v=cv.cuda().view(1, -1, D), length=cfg.cache_len)
    qu = dp.Queue(cfg.n_blocks, cfg.block_rows[0], D)
    for _ in range(cfg.n_blocks):
        dp.queue_push(qu, x["noise"].cuda())
    kv = torch.empty(2, n, D, dtype=torch.float16, device="cuda")
    out = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
    dp.window_step(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), blk, cache, kv, out, H, hd, pop=True, queue=qu,
                   push_noise=x["noise"].cuda())
    dp.device_status()
    rows = sample_rows(cfg.row_offset, n_extra=64)
    mod = O.lookup(x["table"], x["timesteps"])
    want, _, _ = O.window_step(x["q"], x["k"], x["v"], ck, cv, cfg.cache_len, cfg.row_offset,
                               mod, H, hd, rows=rows)
    got = out[rows].cpu().double().numpy()
    assert_close(got, want, "bf16", name)
    n0 = cfg.block_rows[0]
    assert bytes_equal(cache.k[0, :n0], kv[0, :n0]) and bytes_equal(cache.v[0, :n0], kv[1, :n0])
    kr = O.modulate_rounded(x["k"][:n0], [0, n0], mod[:1], "f16")
    assert np.array_equal(cache.k[0, :n0].cpu().double().numpy(), kr)

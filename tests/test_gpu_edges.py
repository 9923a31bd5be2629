"""Edge and maximum sizes of the sublayer kernels, the several-slot attention and the frame
push, through the C ABI against the oracle: one-row and ragged GEMM tiles, the narrowest
output and reduction widths, the widest pre-norm row, sixteen cache slots, sixteen frames."""
import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import assert_close, bytes_equal

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _bf16(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16)


@pytest.mark.parametrize("m,n,k", [(1, 128, 8), (127, 128, 64), (129, 256, 72), (300, 640, 8)])
def test_linear_small_and_ragged(dp, m, n, k):
    a = _bf16((m, k), 1)
    w = _bf16((n, k), 2, std=k ** -0.5)
    bias = torch.randn(n, generator=torch.Generator().manual_seed(3))
    y = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    dp.linear(a.cuda(), w.cuda(), bias.cuda(), y)
    dp.device_status()
    exact = O.linear(a, w, bias)
    bound = 2.0 ** -8 * np.abs(exact) + 2.0 ** -12 * (np.abs(O.as_f64(a)) @ np.abs(O.as_f64(w)).T) + 1e-7
    assert np.all(np.abs(y.cpu().double().numpy() - exact) <= bound)


@pytest.mark.parametrize("hidden,rows", [(8192, [3, 2]), (256, [1])])
def test_ln_modulate_widest_row_and_single_row(dp, hidden, rows):
    x = _bf16((sum(rows), hidden), 4, std=3.0)
    table = torch.tanh(torch.randn(1000, 3, hidden, generator=torch.Generator().manual_seed(5)))
    ts = [1, 998][:len(rows)]
    blk = dp.blocks_from_table(table.cuda(), ts, rows)
    h = torch.empty_like(x, device="cuda")
    dp.ln_modulate(x.cuda(), h, blk)
    dp.device_status()
    want = O.ln_modulate(x, np.cumsum([0] + rows), O.lookup(table, ts), 1e-6)
    assert np.all(np.abs(h.cpu().double().numpy() - want) <= 2.0 ** -8 * np.abs(want) + 1e-6)


def test_sixteen_cache_slots(dp):
    H, hd, cap = 2, 64, 130
    D = H * hd
    rows = [200, 57]
    n = sum(rows)
    g = torch.Generator().manual_seed(6)
    q, k, v = (torch.randn(n, D, generator=g).to(torch.bfloat16) for _ in range(3))
    ring_k = torch.randn(16, cap, D, generator=g).to(torch.float16)
    ring_v = torch.randn(16, cap, D, generator=g).to(torch.float16)
    lens = [cap if s % 3 else (0 if s % 2 else 61) for s in range(16)]   # full, empty and ragged slots
    cache = dp.KVCache(cap, D, torch.float16, n_slots=16, k=ring_k.cuda().clone(), v=ring_v.cuda().clone())
    for s, L in enumerate(lens):
        cache.desc.len[s] = L
    cache.desc.n_advances = 21
    table = torch.tanh(torch.randn(1000, 3, D, generator=g))
    ts = [10, 700]
    blk = dp.blocks_from_table(table.cuda(), ts, rows)
    kv = torch.empty(2, n, D, dtype=torch.float16, device="cuda")
    out = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
    dp.window_step(q.cuda(), k.cuda(), v.cuda(), blk, cache, kv, out, H, hd, cache_all_slots=True)
    dp.device_status()
    ck = torch.cat([ring_k[s, :L] for s, L in enumerate(lens) if L > 0])
    cv = torch.cat([ring_v[s, :L] for s, L in enumerate(lens) if L > 0])
    mod = O.lookup(table, ts)
    ro = [0, rows[0], n]
    # the oracle modulates the raw window k, v itself, in float64
    want, _, _ = O.window_step(q, k, v, ck, cv, ck.shape[0], ro, mod, H, hd)
    assert_close(out.cpu().double().numpy(), want, "bf16", "sixteen slots")


def test_push_sixteen_frames_and_one(dp):
    D, fr = 128, 24
    pool = _bf16((20, fr, D), 7).cuda()
    q = dp.Queue(2, 16 * fr, D)
    idx = [19, 0, 7, 7, 3, 12, 1, 5, 18, 2, 9, 11, 4, 6, 8, 10]      # a frame may repeat within a block
    dp.queue_push_frames(q, pool, idx)
    dp.queue_push_frames(q, pool, [13])
    torch.cuda.synchronize()
    want = torch.cat([pool[i] for i in idx + [13]])
    assert bytes_equal(q.window(), want)
    with pytest.raises(dp.DpError):
        dp.queue_push_frames(dp.Queue(2, 17 * fr, D), pool, list(range(17)))   # more than 16 frames

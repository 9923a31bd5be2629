"""Guard bands around every buffer the library writes, a memory-safety check that needs no
sanitizer: each output lives in the middle of a larger allocation whose head and tail hold a
bit pattern; after the call, on ragged sizes that end in partial tiles, the pattern must be
intact.  Rows of a destination the call is not asked to write (cache-slot rows beyond the
exiting block, queue slots other than the pushed one) are checked the same way."""
import numpy as np
import pytest
import torch

from workloads import make_sublayer_weights

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

G = 8192            # guard elements on each side (16 KiB or more: keeps the middle 16-byte aligned)
PATTERN = {2: 0x5A5A, 4: 0x5A5A5A5A}


class Guarded:
    """A tensor of `shape` inside an allocation with G patterned elements before and after."""

    def __init__(self, shape, dtype):
        self.n = int(np.prod(shape))
        self.buf = torch.empty(self.n + 2 * G, dtype=dtype, device="cuda")
        es = self.buf.element_size()
        self.ibuf = self.buf.view(torch.int16 if es == 2 else torch.int32)
        self.pat = PATTERN[es]
        self.ibuf.fill_(self.pat)
        self.t = self.buf[G:G + self.n].view(*shape)

    def fill(self, value):
        self.t.fill_(value)
        return self

    def intact(self):
        return bool((self.ibuf[:G] == self.pat).all()) and bool((self.ibuf[G + self.n:] == self.pat).all())


def _table(D, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.tanh(torch.randn(1000, 3, D, generator=g)).cuda()


def _rand(shape, seed, dtype=torch.bfloat16, std=0.5):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * std).to(dtype).cuda()


@pytest.mark.parametrize("H,hd,rows,lc", [(2, 64, [200, 101], 77), (3, 128, [129, 1], 300), (2, 64, [1], 0)])
def test_modulate_attention_and_step_stay_inside_their_outputs(dp, H, hd, rows, lc):
    D = H * hd
    n = sum(rows)
    blk = dp.blocks_from_table(_table(D, 1), [0, 999][:len(rows)], rows)
    q, k, v = (_rand((n, D), 2 + i) for i in range(3))
    kf = Guarded((n, D), torch.float16)
    vf = Guarded((n, D), torch.float16)
    dp.adaln_modulate(k, kf.t, blk)
    dp.adaln_modulate(v, vf.t, blk)
    ck, cv = _rand((max(lc, 1), D), 9, torch.float16), _rand((max(lc, 1), D), 10, torch.float16)
    out = Guarded((n, D), torch.bfloat16)
    dp.window_attention(q, kf.t, vf.t, ck, cv, lc, out.t, H, hd, blk, residual=q)
    # the whole step: cache ring (2 slots) and the step's k'/v' scratch guarded
    cap = max(max(rows), lc, 1)
    ring_k = Guarded((2, cap, D), torch.float16).fill(7.0)
    ring_v = Guarded((2, cap, D), torch.float16).fill(7.0)
    cache = dp.KVCache(cap, D, torch.float16, n_slots=2, k=ring_k.t, v=ring_v.t)
    work = Guarded((2 * n * D,), torch.float16)
    out2 = Guarded((n, D), torch.bfloat16)
    dp.window_step(q, k, v, blk, cache, work.t, out2.t, H, hd, pop=True)
    dp.device_status()
    for gbuf in (kf, vf, out, ring_k, ring_v, work, out2):
        assert gbuf.intact()
    # the advance wrote slot 0 rows [0, rows[0]) only
    n0 = rows[0]
    assert bool((ring_k.t[0, n0:] == 7.0).all()) and bool((ring_k.t[1] == 7.0).all())
    assert bool((ring_v.t[0, n0:] == 7.0).all()) and bool((ring_v.t[1] == 7.0).all())
    assert torch.equal(ring_k.t[0, :n0].view(torch.int16), work.t[:n0 * D].view(n0, D).view(torch.int16))


def test_queue_pushes_and_refresh_stay_inside_their_slots(dp):
    D, slot_rows, n_slots = 256, 96, 3
    queue = dp.Queue(n_slots, slot_rows, D)
    lat = Guarded(tuple(queue.latent.shape), torch.bfloat16).fill(3.0)
    queue.latent = lat.t
    queue.desc.latent = lat.t.data_ptr()
    dp.queue_push(queue, _rand((slot_rows, D), 20))
    pool = _rand((6, 16, D), 21)
    dp.queue_push_frames(queue, pool, [5, 0, 2])           # 48 of 96 rows: a short (final) block
    dp.device_status()
    assert lat.intact()
    # the first push wrote physical slot 0 and its mirror (slot 3); the second slot 1 and slot 4, 48 rows
    assert bool((lat.t[2] == 3.0).all()) and bool((lat.t[5] == 3.0).all())
    assert bool((lat.t[1, 48:] == 3.0).all()) and bool((lat.t[4, 48:] == 3.0).all())
    # the fresh-context refresh writes rows [0, n_ctx) of the read slot only
    ring_k = Guarded((2, 128, D), torch.float16).fill(7.0)
    ring_v = Guarded((2, 128, D), torch.float16).fill(7.0)
    cache = dp.KVCache(128, D, torch.float16, n_slots=2, k=ring_k.t, v=ring_v.t)
    x = _rand((77, D), 22)
    dp.context_refresh(x, x, dp.blocks_from_table(_table(D, 23), [0], [77]), cache)
    wts = {key: t.cuda() for key, t in make_sublayer_weights(D, 24).items()}
    scratch = Guarded((77 * D,), torch.bfloat16)
    dp.context_refresh_sublayer(x, dp.blocks_from_table(_table(D, 23), [5], [77]), wts["w_qkv"], wts["b_qkv"],
                                cache, scratch.t)
    dp.device_status()
    for gbuf in (ring_k, ring_v, scratch):
        assert gbuf.intact()
    assert bool((ring_k.t[0, 77:] == 7.0).all()) and bool((ring_k.t[1] == 7.0).all())
    assert bool((ring_v.t[0, 77:] == 7.0).all()) and bool((ring_v.t[1] == 7.0).all())


@pytest.mark.parametrize("m,rows", [(257, [200, 57]), (1, [1])])
def test_sublayer_kernels_stay_inside_their_outputs(dp, m, rows):
    D, H, hd = 512, 4, 128
    wts = {key: t.cuda() for key, t in make_sublayer_weights(D, 30).items()}
    blk = dp.blocks_from_table(_table(D, 31), [0, 999][:len(rows)], rows)
    x = _rand((m, D), 32, std=1.0)
    h = Guarded((m, D), torch.bfloat16)
    dp.ln_modulate(x, h.t, blk)
    y = Guarded((m, 384), torch.float16)
    dp.linear(h.t, wts["w_qkv"][:384], None, y.t)
    q = Guarded((m, D), torch.bfloat16)
    k = Guarded((m, D), torch.float16)
    v = Guarded((m, D), torch.float16)
    dp.qkv_project(h.t, wts["w_qkv"], wts["b_qkv"], q.t, k.t, v.t)
    o = Guarded((m, D), torch.bfloat16)
    dp.out_project(q.t, wts["w_o"], wts["b_o"], blk, x, o.t)
    cache = dp.KVCache(max(rows), D, torch.float16)
    work = Guarded((4 * m * D,), torch.bfloat16)
    out = Guarded((m, D), torch.bfloat16)
    dp.sublayer_step(x, blk, wts["w_qkv"], wts["b_qkv"], wts["w_o"], wts["b_o"], cache, work.t, out.t, H, hd,
                     pop=True)
    dp.device_status()
    for gbuf in (h, y, q, k, v, o, work, out):
        assert gbuf.intact()

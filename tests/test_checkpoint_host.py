"""Checkpoint and restore of a run's state on the host (no GPU): queue and cache descriptors,
their buffers' bytes and the run's progress survive a round trip through torch.save."""
import io

import torch

import long_video_diffusion_b200 as dp


def test_checkpoint_round_trip_is_exact():
    g = torch.Generator().manual_seed(3)
    queue = dp.Queue(5, 64, 128, device="cpu")
    queue.latent.copy_(torch.randn(queue.latent.shape, generator=g).to(torch.bfloat16))
    d = queue.desc
    d.head, d.count, d.n_pushed, d.n_popped = 3, 4, 11, 7
    for i, (r, e) in enumerate([(64, 9), (64, 5), (64, 2), (40, 0)]):
        d.rows[i], d.evals[i] = r, e
    cache = dp.KVCache(64, 128, torch.float16, n_slots=3, device="cpu")
    cache.k.copy_(torch.randn(cache.k.shape, generator=g).half())
    cache.v.copy_(torch.randn(cache.v.shape, generator=g).half())
    cache.desc.len[0], cache.desc.len[1], cache.desc.len[2] = 64, 40, 0
    cache.desc.n_advances = 5
    state = dp.FifoState(step=123, nxt=17, exited_rows=64)

    buf = io.BytesIO()
    torch.save(dp.checkpoint(queue, cache, state), buf)
    buf.seek(0)
    q2, c2, s2 = dp.restore(torch.load(buf), device="cpu")

    assert torch.equal(q2.latent.view(torch.int16), queue.latent.view(torch.int16))
    assert torch.equal(c2.k.view(torch.int16), cache.k.view(torch.int16))
    assert torch.equal(c2.v.view(torch.int16), cache.v.view(torch.int16))
    for f in ("slot_rows", "hidden", "n_slots", "head", "count", "n_pushed", "n_popped", "dtype"):
        assert getattr(q2.desc, f) == getattr(d, f), f
    assert list(q2.desc.rows) == list(d.rows) and list(q2.desc.evals) == list(d.evals)
    for f in ("capacity", "hidden", "n_slots", "n_advances", "dtype"):
        assert getattr(c2.desc, f) == getattr(cache.desc, f), f
    assert list(c2.desc.len) == list(cache.desc.len)
    # the restored descriptors point at the restored buffers, not the saved ones
    assert q2.desc.latent == q2.latent.data_ptr() and c2.desc.k == c2.k.data_ptr() and c2.desc.v == c2.v.data_ptr()
    assert (s2.step, s2.nxt, s2.exited_rows) == (123, 17, 64)
    assert q2.window_rows() == queue.window_rows() and c2.length == cache.length

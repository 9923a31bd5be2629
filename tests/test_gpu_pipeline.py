"""The host-fed StepPipeline (copies on their own streams, overlapped with the compute of the
previous step) gives, step for step, the same bytes as window steps run one after another on
one stream, and leaves the cache and the queue in the same state."""
import pytest
import torch

from tests.gpu_util import bytes_equal
from workloads import as_features, make_step_inputs, step_config

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_pipeline_matches_sequential_steps(dp):
    cfg = step_config("cogvideo_bf16")
    cfg.n_heads = 4
    cfg.block_rows = [512, 512, 512, 300]
    cfg.cache_len = cfg.cache_capacity = 512
    cfg.push_rows = 512
    x = make_step_inputs(cfg)
    H, hd, D, n = cfg.n_heads, cfg.head_dim, cfg.hidden, cfg.n_win
    g = torch.Generator().manual_seed(3)
    steps = [{key: (x[key].float() + 0.01 * s * torch.randn(x[key].shape, generator=g)).to(torch.bfloat16)
              for key in ("q", "k", "v", "noise")} for s in range(5)]
    blk = dp.blocks_from_table(x["table"].cuda(), x["timesteps"], cfg.block_rows)

    def fresh():
        ck, cv = as_features(x["cache_k"], cfg.dtype), as_features(x["cache_v"], cfg.dtype)
        cache = dp.KVCache(cfg.cache_capacity, D, torch.float16, k=ck.cuda().view(1, -1, D).clone(),
                           v=cv.cuda().view(1, -1, D).clone(), length=cfg.cache_len)
        queue = dp.Queue(cfg.n_blocks, 512, D)
        for _ in range(cfg.n_blocks):
            dp.queue_push(queue, x["noise"].cuda())
        return cache, queue, torch.empty(2, n, D, dtype=torch.float16, device="cuda")

    cache_a, queue_a, kv_a = fresh()
    want = []
    for st in steps:
        out = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
        dp.window_step(st["q"].cuda(), st["k"].cuda(), st["v"].cuda(), blk, cache_a, kv_a, out, H, hd, pop=True,
                       queue=queue_a, push_noise=st["noise"].cuda())
        want.append(out.cpu())
    cache_b, queue_b, kv_b = fresh()
    pipe = dp.StepPipeline(n, D, 512)
    pinned = [{key: t.pin_memory() for key, t in st.items()} for st in steps]
    outs = [torch.empty(n, D, dtype=torch.bfloat16).pin_memory() for _ in steps]
    for st, ho in zip(pinned, outs):
        pipe.submit(st["q"], st["k"], st["v"], st["noise"], ho, blk, cache_b, kv_b, H, hd, pop=True, queue=queue_b)
    pipe.finish()
    dp.device_status()
    for s, (w, got) in enumerate(zip(want, outs)):
        assert bytes_equal(got, w), s
    assert bytes_equal(cache_a.k, cache_b.k) and bytes_equal(cache_a.v, cache_b.v)
    assert cache_a.length == cache_b.length and cache_a.n_advances == cache_b.n_advances == 5
    assert bytes_equal(queue_a.window(), queue_b.window())

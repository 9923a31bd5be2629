"""dp_window_step_noalloc: the window step for callers that cannot allocate device memory
(code inside a host that owns all device memory, or loops where cudaMalloc/cudaFree would
synchronize the device).  It must give the regular entry point's results (dp_window_step
with a caller-allocated kv_work) within the bf16 tolerance the other parity tests use, on
two calls in a row: the second call attends to the cache the first one wrote.

This file is collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test."""
import pytest
import torch

from tests.gpu_util import assert_close, bytes_equal
from workloads import as_features, make_step_inputs, step_config

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _state(dp, cfg, x, dev):
    D = cfg.hidden
    cache = dp.KVCache(cfg.cache_capacity, D, torch.float16,
                       k=as_features(x["cache_k"], cfg.dtype).to(dev).view(1, -1, D).clone(),
                       v=as_features(x["cache_v"], cfg.dtype).to(dev).view(1, -1, D).clone(), length=cfg.cache_len)
    queue = dp.Queue(cfg.n_blocks, max(cfg.block_rows), D, device=dev)
    for _ in range(cfg.n_blocks - 1):
        dp.queue_push(queue, x["noise"].to(dev))
    return cache, queue


@pytest.mark.parametrize("shape", [(4, 64, [300, 300, 300, 211]), (12, 128, [1000, 1000, 1000, 1000])],
                         ids=["h4x64_n1111", "h12x128_n4000"])
def test_noalloc_matches_window_step_on_two_calls(dp, shape):
    H, hd, rows = shape
    cfg = step_config("cogvideo_bf16")
    cfg.n_heads, cfg.head_dim, cfg.block_rows = H, hd, rows
    cfg.cache_len = cfg.cache_capacity = cfg.push_rows = max(rows)
    x = make_step_inputs(cfg)
    dev = torch.device("cuda:0")
    D, n = cfg.hidden, cfg.n_win
    assert 2 * n * D * 2 <= dp.NOALLOC_SCRATCH_BYTES
    blk = dp.blocks_from_table(x["table"].to(dev), x["timesteps"], cfg.block_rows)
    q, k, v, noise = (x[key].to(dev) for key in ("q", "k", "v", "noise"))
    cache_a, queue_a = _state(dp, cfg, x, dev)
    cache_b, queue_b = _state(dp, cfg, x, dev)
    kv = torch.empty(2, n, D, dtype=torch.float16, device=dev)
    out_a = torch.empty(n, D, dtype=torch.bfloat16, device=dev)
    out_b = torch.empty_like(out_a)
    for call in range(2):
        dp.window_step(q, k, v, blk, cache_a, kv, out_a, H, hd, pop=True, queue=queue_a, push_noise=noise)
        dp.window_step_noalloc(q, k, v, blk, cache_b, out_b, H, hd, pop=True, queue=queue_b, push_noise=noise)
        dp.device_status()
        assert_close(out_b.cpu().double().numpy(), out_a.cpu().double().numpy(), "bf16", f"call {call}")
        assert cache_b.length == cache_a.length == rows[0]
        assert bytes_equal(cache_b.k[0, :rows[0]], cache_a.k[0, :rows[0]])
        assert bytes_equal(cache_b.v[0, :rows[0]], cache_a.v[0, :rows[0]])
        assert queue_b.count == queue_a.count and queue_b.evals() == queue_a.evals()


def test_noalloc_fp32_window_matches_window_step_and_oracle_on_two_calls(dp):
    """The fp32 path (4-byte features in the fixed array): the tiny fp32 window (2 blocks x
    128 rows, 128-row cache, 2 x 64 heads), two calls in a row, against dp_window_step and
    against the float64 oracle at the fp32 bar."""
    import oracle as O
    cfg = step_config("tiny_f32")
    x = make_step_inputs(cfg)
    dev = torch.device("cuda:0")
    H, hd, D, n = cfg.n_heads, cfg.head_dim, cfg.hidden, cfg.n_win
    blk = dp.blocks_from_table(x["table"].to(dev), x["timesteps"], cfg.block_rows)
    q, k, v, noise = (x[key].to(dev) for key in ("q", "k", "v", "noise"))

    def state():
        cache = dp.KVCache(cfg.cache_capacity, D, torch.float32, k=x["cache_k"].to(dev).view(1, -1, D).clone(),
                           v=x["cache_v"].to(dev).view(1, -1, D).clone(), length=cfg.cache_len)
        queue = dp.Queue(cfg.n_blocks, max(cfg.block_rows), D, dtype=torch.float32, device=dev)
        for _ in range(cfg.n_blocks - 1):
            dp.queue_push(queue, noise)
        return cache, queue

    cache_a, queue_a = state()
    cache_b, queue_b = state()
    kv = torch.empty(2, n, D, dtype=torch.float32, device=dev)
    out_a = torch.empty(n, D, dtype=torch.float32, device=dev)
    out_b = torch.empty_like(out_a)
    mod = O.lookup(x["table"], x["timesteps"])
    ck, cv, L = x["cache_k"], x["cache_v"], cfg.cache_len
    for call in range(2):
        dp.window_step(q, k, v, blk, cache_a, kv, out_a, H, hd, pop=True, queue=queue_a, push_noise=noise)
        dp.window_step_noalloc(q, k, v, blk, cache_b, out_b, H, hd, pop=True, queue=queue_b, push_noise=noise)
        dp.device_status()
        got = out_b.cpu().double().numpy()
        assert_close(got, out_a.cpu().double().numpy(), "f32", f"call {call} vs dp_window_step")
        want, kp, vp = O.window_step(x["q"], x["k"], x["v"], ck, cv, L, cfg.row_offset, mod, H, hd)
        assert_close(got, want, "f32", f"call {call} vs the oracle")
        n0 = cfg.block_rows[0]
        assert cache_b.length == cache_a.length == n0
        assert bytes_equal(cache_b.k[0, :n0], cache_a.k[0, :n0])
        assert bytes_equal(cache_b.v[0, :n0], cache_a.v[0, :n0])
        assert queue_b.count == queue_a.count and queue_b.evals() == queue_a.evals()
        # the second call attends to the cache the first one wrote: the head block's k', v'
        ck, cv, L = cache_b.k[0, :n0].cpu(), cache_b.v[0, :n0].cpu(), n0


def test_noalloc_rejects_windows_beyond_its_scratch(dp):
    H, hd = 16, 128
    n = dp.NOALLOC_SCRATCH_BYTES // (2 * H * hd * 2) + 1   # one row too many
    dev = torch.device("cuda:0")
    table = torch.zeros(1, 3, H * hd, device=dev)
    blk = dp.blocks_from_table(table, [0], [n])
    q = torch.zeros(n, H * hd, dtype=torch.bfloat16, device=dev)
    out = torch.empty_like(q)
    cache = dp.KVCache(8, H * hd, torch.float16, device=dev)
    with pytest.raises(dp.DpError) as e:
        dp.window_step_noalloc(q, q, q, blk, cache, out, H, hd)
    assert e.value.status == dp.ERR_CAPACITY and "scratch" in str(e.value)
    assert cache.n_advances == 0

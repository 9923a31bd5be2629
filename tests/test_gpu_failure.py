"""Failure detection of the tensor-core attention without a GPU fault: with the
DP_TEST_SKIP_KV_LOADS hook the producer issues no loads, every wait for them gives up at
its bound (about 2 s of SM clock), the kernel releases its resources and returns, the host
reads DP_ERR_TIMEOUT from the device status word, and the context stays usable."""
import time

import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import assert_close
from workloads import to_dtype

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _inputs(n, H, hd, seed=7):
    g = torch.Generator().manual_seed(seed)
    D = H * hd
    q = to_dtype(torch.randn(n, D, generator=g), "bf16")
    k, v = (to_dtype(torch.randn(n, D, generator=g), "bf16").to(torch.float16) for _ in range(2))
    table = torch.tanh(torch.randn(4, 3, D, generator=g))
    return q, k, v, table


@pytest.mark.parametrize("hd", [64, 128])
def test_bounded_wait_reports_timeout_and_context_survives(dp, hd):
    H, n = 1, 200                      # one CTA: 256 query rows of one head
    q, k, v, table = _inputs(n, H, hd)
    blk = dp.blocks_from_table(table.cuda(), [1, 3], [120, 80])
    out = torch.full((n, H * hd), 7.0, dtype=torch.bfloat16, device="cuda")
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    dp.device_status()                  # clean slate
    t0 = time.time()
    dp.window_attention(qd, kd, vd, None, None, 0, out, H, hd, blk,
                        flags=dp.MOD_Q | dp.GATE_OUT | dp.TEST_SKIP_KV_LOADS)
    with pytest.raises(dp.DpError) as e:
        dp.device_status()
    elapsed = time.time() - t0
    assert e.value.status == dp.ERR_TIMEOUT
    assert 0.5 < elapsed < 60.0
    assert bool((out == 7.0).all())     # nothing was written
    dp.device_status()                  # the status word was cleared
    # the context is still usable: a normal call gives the right answer
    dp.window_attention(qd, kd, vd, None, None, 0, out, H, hd, blk)
    dp.device_status()
    want = O.window_attention(q, k, v, np.zeros((0, H * hd)), np.zeros((0, H * hd)), 0, blk.offsets,
                              O.lookup(table, [1, 3]), H, hd)
    assert_close(out.cpu().double().numpy(), want, "bf16", "after timeout")

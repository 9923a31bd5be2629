"""Shared helpers for the GPU parity tests (CUDA path vs the CPU oracle on the same
seeded inputs).  Tolerances are the acceptance bar of the window step: fp32 max-abs 1e-4;
bf16 max-abs 2e-2 and relative L2 5e-3 (fp32 accumulation); copies bit-exact."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O

TOL = {"f32": {"max_abs": 1e-4, "rel_l2": None}, "bf16": {"max_abs": 2e-2, "rel_l2": 5e-3}}


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the CUDA result"
    d = got - ref
    max_abs = float(np.max(np.abs(d))) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300)) if d.size else 0.0
    return max_abs, rel


def assert_close(got, ref, dtype: str, what: str = ""):
    max_abs, rel = errors(got, ref)
    tol = TOL[dtype]
    assert max_abs <= tol["max_abs"], f"{what}: max-abs {max_abs:.3e} > {tol['max_abs']}"
    if tol["rel_l2"] is not None:
        assert rel <= tol["rel_l2"], f"{what}: rel-L2 {rel:.3e} > {tol['rel_l2']}"
    return max_abs, rel


def sample_rows(row_offset, n_extra: int = 96, seed: int = 0):
    """First and last rows, both sides of every block boundary, the last 128-row tile
    (ragged tail), and seeded random rows."""
    n = row_offset[-1]
    rows = {0, n - 1}
    for b in row_offset[1:-1]:
        for r in (b - 1, b, b + 1):
            if 0 <= r < n:
                rows.add(r)
    tail0 = (n - 1) // 256 * 256
    for r in range(tail0, n, max(1, (n - tail0) // 8)):
        rows.add(r)
    rng = np.random.default_rng(seed)
    rows.update(int(x) for x in rng.integers(0, n, size=n_extra))
    return sorted(rows)


def bytes_equal(a: torch.Tensor, b: torch.Tensor) -> bool:
    if a.shape != b.shape or a.dtype != b.dtype:
        return False
    return bool(torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8)))


def cuda_sync():
    torch.cuda.synchronize()

"""The FMA-pipe exp2 used for part of the softmax: its coefficients are the committed fit's,
and an emulation of the kernel's float32 steps (round-to-integer by adding 1.5 * 2^23, the
degree-3 polynomial on the remainder, the integer added to the exponent field) stays within
the fit's relative error bound over the range the softmax produces (x in [-125, 8])."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "long_video_diffusion_b200", "csrc")


def _fit():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.float32_coeffs()


def _kernel_coeffs():
    src = open(os.path.join(CSRC, "dp_attn_tc.cu")).read()
    return [np.float32(float(re.search(rf"kPolyC{i} = ([0-9.e+-]+)f;", src).group(1))) for i in range(4)]


def _fma32(a, b, c):
    # a float32 fused multiply-add: the float64 product of float32 values is exact
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _emulate(x):
    c0, c1, c2, c3 = [np.full_like(x, v) for v in _kernel_coeffs()]
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    r = (t - np.float32(12582912.0)).astype(np.float32)
    f = _fma32(r, np.full_like(x, -1.0), x)
    q = _fma32(c3, f, c2)
    q = _fma32(q, f, c1)
    q = _fma32(q, f, c0)
    bits = (q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_kernel_coefficients_are_the_fit():
    c32, err, err32 = _fit()
    assert [float(v) for v in c32] == [float(v) for v in _kernel_coeffs()]
    assert err32 < 8e-5


def test_emulated_exp2_within_bound():
    _, _, err32 = _fit()
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32),
                        np.arange(-125, 9, dtype=np.float32),
                        np.arange(-125, 8, dtype=np.float32) + np.float32(0.5)])
    got = _emulate(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert float(rel.max()) <= err32 + 2e-7      # + float32 evaluation rounding
    assert np.all(got > 0) and np.all(np.isfinite(got))


def test_masked_keys_underflow_to_zero_weight():
    got = _emulate(np.array([-np.inf, -1e30, -126.0], dtype=np.float32))
    assert np.all(got <= 2.0 ** -124) and np.all(got >= 0)

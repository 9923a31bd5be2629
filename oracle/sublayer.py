"""Plain float64 definitions of the DiT attention sublayer around the window attention
(test infrastructure only; see the package docstring for who may import it).

Sources (page title, then the part of it):
  [A]  "Minute-Long Videos with Dual Parallelisms" (arXiv 2505.21070), abstract: the
       denoiser is a Diffusion Transformer; a feature cache reuses the prior block's
       features as context.
  [R2] pith.science review of 2505.21070, referee major comment on Section 3.2: the cache
       holds the self-attention K and V features of the neighbouring block.
  [R3] same review, supporting citations: DiT-style conditioning of every block on its own
       timestep.

Readings where the pages are silent:
  * the sublayer is the DiT self-attention sublayer with adaLN conditioning:
        h   = LN(x) * (1 + scale_b) + shift_b          (LN without affine parameters)
        q, k, v = h W_qkv^T + b_qkv                     (W: out-features x in-features)
        o   = softmax(q K^T / sqrt(head_dim)) V over [cache ; window]
        out = x + gate_b * (o W_o^T + b_o)
    with b the block of the row; LN's variance is the biased one (mean of squared
    deviations) and eps is added under the square root.
  * the cache holds the projected k and v of the exited block (the self-attention
    features [R2]); nothing is recomputed for cached rows.
  * ``rounded=True`` stores the intermediates the way a 16-bit pipeline does: h, q and o
    in bf16, k and v in f16 (saturating at +-65504), each rounded once to nearest even
    from the float64 value.  The float64 arithmetic in between is unchanged.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

from .dualparal import as_f64, row_blocks, window_attention


def round_to(x, dtype: str) -> np.ndarray:
    """Round float64 values once to ``dtype`` ("bf16", "f16" saturating, "f32"); return
    the stored values as float64."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(as_f64(x)))
    if dtype == "bf16":
        return t.to(torch.bfloat16).to(torch.float64).numpy()
    if dtype == "f16":
        return t.clamp(-65504.0, 65504.0).to(torch.float16).to(torch.float64).numpy()
    if dtype == "f32":
        return t.to(torch.float32).to(torch.float64).numpy()
    raise ValueError(dtype)


def layer_norm(x, eps: float) -> np.ndarray:
    """(x - mean) / sqrt(var + eps) per row, mean and biased variance over the channels."""
    x = as_f64(x)
    mean = x.mean(axis=1, keepdims=True)
    d = x - mean
    var = (d * d).mean(axis=1, keepdims=True)
    return d / np.sqrt(var + eps)


def ln_modulate(x, row_offset: Sequence[int], mod, eps: float) -> np.ndarray:
    """h[i] = LN(x[i]) * (1 + scale_b) + shift_b, b = block of row i [R3]."""
    n = layer_norm(x, eps)
    mod = as_f64(mod)
    beta = row_blocks(row_offset, n.shape[0])
    return n * (1.0 + mod[beta, 1, :]) + mod[beta, 0, :]


def linear(a, w, bias=None) -> np.ndarray:
    """a W^T + bias; W is [out_features][in_features]."""
    y = as_f64(a) @ as_f64(w).T
    if bias is not None:
        y = y + as_f64(bias)[None, :]
    return y


def sublayer_step(x, w_qkv, b_qkv, w_o, b_o, cache_k, cache_v, cache_len: int,
                  row_offset: Sequence[int], mod, n_heads: int, head_dim: int, eps: float, *,
                  rounded: bool = True, rows: Optional[Sequence[int]] = None):
    """One sublayer step on the window x [n_win, D].  Returns (out, k, v): out for the
    query rows ``rows`` (all rows if None), and the window's projected k and v (all rows)
    as they enter the attention and the cache."""
    x = as_f64(x)
    n_win, D = x.shape
    if D != n_heads * head_dim:
        raise ValueError("hidden != n_heads * head_dim")
    h = ln_modulate(x, row_offset, mod, eps)
    if rounded:
        h = round_to(h, "bf16")
    qkv = linear(h, w_qkv, b_qkv)
    q, k, v = qkv[:, :D], qkv[:, D:2 * D], qkv[:, 2 * D:]
    if rounded:
        q, k, v = round_to(q, "bf16"), round_to(k, "f16"), round_to(v, "f16")
    sel = np.arange(n_win) if rows is None else np.asarray(rows, dtype=np.int64)
    o = window_attention(q, k, v, cache_k, cache_v, cache_len, row_offset, mod, n_heads, head_dim,
                         mod_q=False, gate_out=False, rows=None if rows is None else sel)
    if rounded:
        o = round_to(o, "bf16")
    mod = as_f64(mod)
    beta = row_blocks(row_offset, n_win)
    out = x[sel] + mod[beta[sel], 2, :] * linear(o, w_o, b_o)
    return out, k, v


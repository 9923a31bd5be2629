"""Plain float64 definitions of the fresh-context variant of the feature cache (test
infrastructure only; see the package docstring for who may import it).

Sources (page title, then the part of it):
  [R2] pith.science review of "Minute-Long Videos with Dual Parallelisms" (arXiv
       2505.21070), referee major comment on Section 3.2: the cache reuses the context
       block's self-attention K and V from one denoising step earlier; the referee asks for
       an ablation against K and V recomputed at the current step.
  [R4] same review, skeptic's concrete test: a run with the feature cache masked, to isolate
       the effect of reusing stale K/V.

Reading where the pages are silent:
  * "recomputed" means: the context block's K and V are produced again, at the step that
    uses them, from the context rows and the conditioning the caller gives for that step,
    by the same projection the window's own rows go through -- the identity projection with
    adaLN modulation of the window step, or pre-norm + modulation + the k/v rows of the
    q/k/v projection in the DiT sublayer.  The cached variant instead stores what the
    block's last evaluation produced.
  * the context rows carry a block table of their own (usually one block); its modulation
    vectors are those of the timestep the caller conditions the context on.
"""
from __future__ import annotations

from typing import Sequence, Tuple

import numpy as np

from .dualparal import as_f64, modulate
from .sublayer import linear, ln_modulate, round_to


def fresh_context(k_ctx, v_ctx, row_offset: Sequence[int], mod) -> Tuple[np.ndarray, np.ndarray]:
    """Window-step features of the context rows, recomputed now [R2]: k' = k (1 + scale_b) +
    shift_b and v' likewise, b = the context block of the row.  Returns (k', v') in float64."""
    return modulate(k_ctx, row_offset, mod), modulate(v_ctx, row_offset, mod)


def fresh_context_sublayer(x_ctx, row_offset: Sequence[int], mod, w_qkv, b_qkv, eps: float, *,
                           rounded: bool = True) -> Tuple[np.ndarray, np.ndarray]:
    """Sublayer features of the context rows, recomputed now [R2]: h = LN(x) (1 + scale_b) +
    shift_b, then k = h W_k^T + b_k and v = h W_v^T + b_v with W_k, W_v the second and third
    thirds of the rows of W_qkv (and of b_qkv).  ``rounded`` stores h in bf16 and k, v in f16
    the way the 16-bit pipeline does."""
    x = as_f64(x_ctx)
    D = x.shape[1]
    h = ln_modulate(x, row_offset, mod, eps)
    if rounded:
        h = round_to(h, "bf16")
    w = as_f64(w_qkv)
    b = None if b_qkv is None else as_f64(b_qkv)
    k = linear(h, w[D:2 * D], None if b is None else b[D:2 * D])
    v = linear(h, w[2 * D:3 * D], None if b is None else b[2 * D:3 * D])
    if rounded:
        k, v = round_to(k, "f16"), round_to(v, "f16")
    return k, v

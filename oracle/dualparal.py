"""Plain float64 definitions of the DualParal window step (test infrastructure only).

Sources (page title, then the part of it):
  [A]  "Minute-Long Videos with Dual Parallelisms" (arXiv 2505.21070), abstract: frame
       blocks processed with progressively decreasing noise levels; a feature cache that
       stores and reuses features of the prior block as context.
  [R1] pith.science review of 2505.21070, key machinery / referee summary (Section 3.1,
       Figure 1): a FIFO queue, noise levels decreasing from tail to head; each step
       appends a noisy block at the tail and pops a clean block at the head.
  [R2] same review, referee major comment on Section 3.2: the cache holds the
       self-attention K and V features of the neighbouring block, computed one
       denoising step earlier.
  [R3] same review, supporting citation of DiT-style conditioning (the model is a
       Diffusion Transformer whose blocks are conditioned on their own timestep).

Readings where the pages are silent:
  * adaLN modulation is y = x * (1 + scale_b) + shift_b, per channel, with (shift, scale,
    gate) the rows of a per-timestep table; the gate multiplies the attention output.
  * q, k and v of the window are modulated with their own block's vectors; cached K/V are
    stored features and are not modulated again.
  * attention is bidirectional over [cache rows 0..L_c ; all window rows], softmax scale
    1/sqrt(head_dim); nothing is masked except rows beyond the valid lengths.
  * head block (smallest timestep, cleanest) first; the head block exits; its K'/V' from
    its last evaluation become the cache.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import numpy as np


def as_f64(x) -> np.ndarray:
    """Exact upcast of a torch tensor (fp32/bf16) or array to a float64 ndarray."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _check_offsets(row_offset: Sequence[int], n_rows: int) -> np.ndarray:
    ro = np.asarray(row_offset, dtype=np.int64)
    if ro.ndim != 1 or ro.size < 2 or ro[0] != 0 or ro[-1] != n_rows or np.any(np.diff(ro) < 0):
        raise ValueError(f"bad row_offset {list(ro)} for {n_rows} rows")
    return ro


def row_blocks(row_offset: Sequence[int], n_rows: int) -> np.ndarray:
    """beta(i): the block that owns window row i (blocks are contiguous row ranges)."""
    ro = _check_offsets(row_offset, n_rows)
    beta = np.empty(n_rows, dtype=np.int64)
    for b in range(ro.size - 1):
        beta[ro[b]:ro[b + 1]] = b
    return beta


def lookup(table, timesteps: Sequence[int]) -> np.ndarray:
    """Per-block (shift, scale, gate) = table[t_b]; [B, 3, D].  Stands in for the DiT's
    timestep MLP [R3]; each block is conditioned on its own staggered timestep [R1]."""
    tab = as_f64(table)
    return np.stack([tab[int(t)] for t in timesteps], axis=0)


def modulate(x, row_offset: Sequence[int], mod) -> np.ndarray:
    """y[i, c] = x[i, c] * (1 + scale_beta(i)[c]) + shift_beta(i)[c]   (float64)."""
    x = as_f64(x)
    mod = as_f64(mod)
    beta = row_blocks(row_offset, x.shape[0])
    shift = mod[beta, 0, :]
    scale = mod[beta, 1, :]
    return x * (1.0 + scale) + shift


def modulate_rounded(x, row_offset: Sequence[int], mod, dtype: str) -> np.ndarray:
    """The modulated features as stored in ``dtype`` ("f32", "bf16" or "f16"): 1 + scale is
    formed in float32, the product and sum are exact in float64 (at most 11-bit x 24-bit
    significands), then the value is rounded once to float32 and once more to the storage
    type (round to nearest even; f16 saturates at +-65504 instead of overflowing).
    Returns the stored values as float64."""
    import torch
    x = as_f64(x)
    mod = as_f64(mod).astype(np.float32)
    beta = row_blocks(row_offset, x.shape[0])
    a = (np.float32(1.0) + mod[:, 1, :]).astype(np.float64)      # fp32 add, RNE
    y = x * a[beta] + mod[beta, 0, :].astype(np.float64)
    y32 = torch.from_numpy(y.astype(np.float32))
    if dtype == "f32":
        return y32.to(torch.float64).numpy()
    if dtype == "bf16":
        return y32.to(torch.bfloat16).to(torch.float64).numpy()
    if dtype == "f16":
        return y32.clamp(-65504.0, 65504.0).to(torch.float16).to(torch.float64).numpy()
    raise ValueError(dtype)


def window_attention(q, k, v, cache_k, cache_v, cache_len: int, row_offset: Sequence[int],
                     mod, n_heads: int, head_dim: int, *, mod_q: bool = True,
                     gate_out: bool = True, residual=None, softmax_scale: Optional[float] = None,
                     rows: Optional[Sequence[int]] = None, q_chunk: int = 512) -> np.ndarray:
    """Window attention over [cached K/V ; window K/V] [A][R2].

    q: window queries [n_win, D] (raw; modulated here when mod_q).  k, v: the window's
    keys/values as they enter attention (already modulated by the caller).  cache_k/v:
    [capacity, D], rows 0..cache_len valid.  Per head h and query row i:
        s_ij = (q'_i . K_j) * softmax_scale,  p_ij = exp(s_ij - max_j s_ij) / sum_j(...)
        o_i  = sum_j p_ij V_j;  out_i = gate_beta(i) * o_i (+ residual_i)
    ``rows`` restricts the computation to a subset of query rows (returned in that order).
    """
    n_win, D = q.shape
    if D != n_heads * head_dim:
        raise ValueError("hidden != n_heads * head_dim")
    mod = as_f64(mod)
    beta = row_blocks(row_offset, n_win)
    sel = np.arange(n_win) if rows is None else np.asarray(rows, dtype=np.int64)
    qs = as_f64(q[sel] if rows is not None else q)
    if mod_q:
        qs = qs * (1.0 + mod[beta[sel], 1, :]) + mod[beta[sel], 0, :]
    # keys and values: [cache rows 0..L_c ; window rows], laid out head-major [H, L, hd]
    K = np.concatenate([as_f64(cache_k[:cache_len]), as_f64(k)], axis=0)
    V = np.concatenate([as_f64(cache_v[:cache_len]), as_f64(v)], axis=0)
    L = K.shape[0]
    Kh_all = np.ascontiguousarray(K.reshape(L, n_heads, head_dim).transpose(1, 0, 2))
    Vh_all = np.ascontiguousarray(V.reshape(L, n_heads, head_dim).transpose(1, 0, 2))
    del K, V
    scale = (1.0 / math.sqrt(head_dim)) if softmax_scale is None else float(softmax_scale)
    out = np.empty((sel.size, D), dtype=np.float64)
    for h in range(n_heads):
        c0, c1 = h * head_dim, (h + 1) * head_dim
        Kh = Kh_all[h]
        Vh = Vh_all[h]
        for r0 in range(0, sel.size, q_chunk):
            qh = qs[r0:r0 + q_chunk, c0:c1]
            s = (qh @ Kh.T) * scale                 # pass 1: logits and row max
            m = s.max(axis=1, keepdims=True)
            p = np.exp(s - m)                       # pass 2: exponentials, sum, weights
            p /= p.sum(axis=1, keepdims=True)
            out[r0:r0 + q_chunk, c0:c1] = p @ Vh
    if gate_out:
        out *= mod[beta[sel], 2, :]
    if residual is not None:
        out += as_f64(residual)[sel]
    return out


def window_step(q, k, v, cache_k, cache_v, cache_len: int, row_offset: Sequence[int], mod,
                n_heads: int, head_dim: int, *, residual=None,
                rows: Optional[Sequence[int]] = None):
    """One window step: K/V modulation, then attention with the Q prologue and gate
    epilogue.  Returns (out, k', v') with k', v' the window's modulated features."""
    kp = modulate(k, row_offset, mod)
    vp = modulate(v, row_offset, mod)
    out = window_attention(q, kp, vp, cache_k, cache_v, cache_len, row_offset, mod,
                           n_heads, head_dim, residual=residual, rows=rows)
    return out, kp, vp


# ----------------------------------------------------------------------------- queue state

class KVCacheRing:
    """Feature cache [R2]: a ring of ``n_slots`` slots of ``capacity`` rows; the advance
    writes the exiting block's K'/V' into slot ``n_advances mod n_slots``."""

    def __init__(self, n_slots: int, capacity: int, hidden: int, k=None, v=None,
                 length: int = 0):
        self.n_slots = n_slots
        self.capacity = capacity
        self.k = np.zeros((n_slots, capacity, hidden))
        self.v = np.zeros((n_slots, capacity, hidden))
        if k is not None:
            self.k[0] = as_f64(k)
            self.v[0] = as_f64(v)
        self.len = [length] + [0] * (n_slots - 1)
        self.n_advances = 0

    def advance(self, k_exit, v_exit, n_exit: int) -> int:
        if n_exit > self.capacity:
            raise ValueError("exiting block larger than the cache slot")
        slot = self.n_advances % self.n_slots
        self.k[slot, :n_exit] = as_f64(k_exit)[:n_exit]
        self.v[slot, :n_exit] = as_f64(v_exit)[:n_exit]
        self.len[slot] = n_exit
        self.n_advances += 1
        return slot

    def latest(self):
        """The most recently written slot (the one attention reads)."""
        slot = (self.n_advances - 1) % self.n_slots if self.n_advances else 0
        return self.k[slot], self.v[slot], self.len[slot]


@dataclass
class _Block:
    ident: int
    latent: np.ndarray
    evals: int = 0


class FifoQueue:
    """The block queue [R1]: blocks ordered head (cleanest) to tail (noisiest)."""

    def __init__(self, max_blocks: int):
        self.max_blocks = max_blocks
        self.blocks: List[_Block] = []
        self.pushed = 0
        self.popped = 0

    def push(self, latent, ident: Optional[int] = None) -> None:
        if len(self.blocks) >= self.max_blocks:
            raise ValueError("queue full")
        self.blocks.append(_Block(self.pushed if ident is None else ident,
                                  as_f64(latent).copy()))
        self.pushed += 1

    def pop(self) -> _Block:
        if not self.blocks:
            raise ValueError("queue empty")
        self.popped += 1
        return self.blocks.pop(0)

    def window(self) -> np.ndarray:
        return np.concatenate([b.latent for b in self.blocks], axis=0)

    def row_offset(self) -> List[int]:
        out = [0]
        for b in self.blocks:
            out.append(out[-1] + b.latent.shape[0])
        return out

    def mark_evaluated(self) -> None:
        for b in self.blocks:
            b.evals += 1


# ----------------------------------------------------------------------------- long run

def entry_step(b: int, n_timesteps: int, window_blocks: int) -> int:
    """Step at which block b enters: floor(b * T / W), so exactly W blocks are live in the
    steady state and the exit of block b coincides with the entry of block b + W."""
    return (b * n_timesteps) // window_blocks


def timestep_schedule(n_timesteps: int, t_max: int = 999) -> List[int]:
    """tau[k] = round(t_max * (1 - k / (T - 1))): noisiest first (k = 0 is t_max)."""
    return [int(round(t_max * (1.0 - k / (n_timesteps - 1)))) for k in range(n_timesteps)]


def long_run_schedule(n_blocks: int, window_blocks: int, n_timesteps: int) -> List[Dict]:
    """Per step s: live blocks (head first) with their evaluation index, and the blocks
    popped (after their last evaluation) and pushed (for the next step) at its end."""
    e = [entry_step(b, n_timesteps, window_blocks) for b in range(n_blocks)]
    total = e[-1] + n_timesteps
    steps = []
    for s in range(total):
        live = [b for b in range(n_blocks) if e[b] <= s < e[b] + n_timesteps]
        steps.append({
            "step": s,
            "live": live,
            "k": [s - e[b] for b in live],
            "pop_after": [b for b in live if s - e[b] == n_timesteps - 1],
            "push_after": [b for b in range(n_blocks) if e[b] == s + 1],
        })
    return steps


class LongRun:
    """Oracle view of the long-video queue run at any step (latents do not change between
    steps: the denoiser update needs the trained model, so q = k = v = the block latent).

    ``noise``: list of per-block latents (entry order); ``table``: [1000, 3, D];
    ``tau``: timestep of evaluation index k.  ``context_blocks``: how many of the most
    recently exited blocks the cache holds and attention reads (1 = the block that just
    left [R2]; more is the NumC context of several exited blocks)."""

    def __init__(self, noise: Sequence, table, n_heads: int, head_dim: int,
                 window_blocks: int, n_timesteps: int, context_blocks: int = 1):
        self.noise = list(noise)
        self.table = as_f64(table)
        self.n_heads = n_heads
        self.head_dim = head_dim
        self.W = window_blocks
        self.T = n_timesteps
        self.tau = timestep_schedule(n_timesteps)
        self.schedule = long_run_schedule(len(self.noise), window_blocks, n_timesteps)
        self.C = int(context_blocks)

    def step_inputs(self, s: int):
        st = self.schedule[s]
        lat = [as_f64(self.noise[b]) for b in st["live"]]
        x = np.concatenate(lat, axis=0)
        ro = [0]
        for a in lat:
            ro.append(ro[-1] + a.shape[0])
        t = [self.tau[k] for k in st["k"]]
        mod = lookup(self.table, t)
        # cache: the K'/V' of the most recently exited block(s), each from its last evaluation
        exited = [b for b in range(len(self.noise))
                  if any(b in self.schedule[u]["pop_after"] for u in range(s))]
        if exited:
            m_last = lookup(self.table, [self.tau[self.T - 1]])
            parts = []
            for b in exited[-self.C:]:
                n = as_f64(self.noise[b])
                parts.append(modulate(n, [0, n.shape[0]], m_last))
            ck = np.concatenate(parts, axis=0)
            cv = ck.copy()
            L = ck.shape[0]
        else:
            ck = np.zeros((0, x.shape[1]))
            cv = ck
            L = 0
        return x, ro, t, mod, ck, cv, L

    def step(self, s: int, rows: Optional[Sequence[int]] = None):
        x, ro, t, mod, ck, cv, L = self.step_inputs(s)
        out, kp, vp = window_step(x, x, x, ck, cv, L, ro, mod, self.n_heads, self.head_dim,
                                  rows=rows)
        return out, ro, t, L

"""Coordinated noise initialisation of the block queue, as a plain definition (test
infrastructure only; see the package docstring for who may import it).

Sources (page title, then the part of it):
  [A]  "Minute-Long Videos with Dual Parallelisms" (arXiv 2505.21070), abstract: a
       coordinated noise initialisation shares initial noise patterns across devices,
       giving globally consistent temporal dynamics at no extra cost.
  [R4] pith.science review of 2505.21070: each new block is drawn from the full noise
       space while shuffling, so that concatenated blocks do not reuse identical noise
       patterns; the recipe is a full noise pool, shuffled assignment and the exclusion of
       the last few latents.

Reading where the pages are silent: the pool is the initial
noise of the first window, one independent N(0, 1) draw per latent frame; the first
window's blocks take the pool's frames in order; every later block takes its frames from
the pool in the order of a fresh random permutation, skipping the frames of the block just
before it (the last latents before it in the video), so adjacent blocks never share a noise
frame.  The permutations are inputs (the random numbers of the method).
"""
from __future__ import annotations

from typing import List, Sequence

import numpy as np

from .dualparal import as_f64


def coordinated_frames(pool_frames: int, block_frames: int, prev_frames: Sequence[int],
                       perm: Sequence[int]) -> List[int]:
    """The pool frames of a new block: perm's order, the previous block's frames skipped,
    the first block_frames of what is left."""
    if sorted(perm) != list(range(pool_frames)):
        raise ValueError("perm is not a permutation of the pool's frames")
    excluded = set(int(f) for f in prev_frames)
    if pool_frames - len(excluded) < block_frames:
        raise ValueError("pool too small for a block that avoids the previous block's frames")
    picked = [int(f) for f in perm if int(f) not in excluded]
    return picked[:block_frames]


def coordinated_schedule(block_frames: Sequence[int], window_blocks: int,
                         perms: Sequence[Sequence[int]]) -> List[List[int]]:
    """Pool frames of every block of a video whose block b has block_frames[b] latent frames;
    the pool is the first window (window_blocks blocks).  perms[b] is block b's permutation
    (used for b >= window_blocks)."""
    W = window_blocks
    pool_frames = int(sum(block_frames[:W]))
    out: List[List[int]] = []
    f0 = 0
    for b, nf in enumerate(block_frames):
        if b < W:
            out.append(list(range(f0, f0 + nf)))
            f0 += nf
        else:
            out.append(coordinated_frames(pool_frames, nf, out[b - 1], perms[b]))
    return out


def gather_frames(pool, frames: Sequence[int]) -> np.ndarray:
    """The latent rows of a block made of pool frames (pool: [frames, frame_rows, D])."""
    p = as_f64(pool)
    return np.concatenate([p[f] for f in frames], axis=0)

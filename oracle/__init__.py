"""CPU oracle for the DualParal window step — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline leg and its
``--impl reference`` arm) may import this package.  The product path
(``long_video_diffusion_b200``) never imports, calls or executes anything here, and this
package imports nothing from it: the two share no code.  The only shared module is
``workloads`` (seeded input draws, none of the method's arithmetic).

Everything is plain NumPy in float64 (inputs are bf16/fp32 values upcast exactly), written
from the definitions in "Minute-Long Videos with Dual Parallelisms" (arXiv 2505.21070):
the abstract's block-wise queue at decreasing noise levels and its feature cache of the
prior block, and the review's account of the cache (Section 3.2: self-attention K/V
features of the neighbouring block, one step stale) and of the FIFO queue (Section 3.1,
Figure 1: push a noisy block at the tail, pop a clean block at the head).

Parity status of each function (how it is pinned, in tests/test_oracle_pins.py):
  lookup            pinned: direct indexing special cases
  modulate          pinned: zero shift/scale -> identity; scale = -1 -> shift_b per block
  modulate_rounded  pinned: equals modulate within one bf16 rounding; bit pattern of
                    hand-computed cases
  window_attention  pinned: brute-force loops on tiny inputs; closed forms (two keys,
                    one key, identical keys, V = 1); torch SDPA reduction; permutation
                    invariance; masked cache rows have no effect; gate = 0 -> residual
  window_step       pinned through its parts and the SDPA reduction
  KVCacheRing / FifoQueue / advance
                    pinned: structural invariants (one push and one pop per advance,
                    cache after k advances = k-th exited block, bytes preserved)
  long_run_schedule pinned: every block evaluated exactly T times in timestep order,
                    at most W live, exit of block b coincides with entry of b + W,
                    noise level monotone along the queue
  layer_norm        pinned: hand-computed row; zero mean and variance var/(var + eps);
                    a constant row maps to zero; brute-force loops
  ln_modulate       pinned: zero shift/scale -> layer_norm; scale = -1 -> shift_b
  linear            pinned: brute-force loops; identity weights -> a + bias
  round_to          pinned: hand-computed bf16/f16 bit patterns, f16 saturation
  sublayer_step     pinned: identity projections reduce it to x + gated window_attention
                    of the normed window; brute-force loops end to end on tiny inputs
  fresh_context / fresh_context_sublayer
                    pinned: equal to the window step's and the sublayer step's own
                    features of the same rows; zero shift/scale -> the rows; a
                    hand-computed LN + projection; the long run's cache at its final
                    timestep
  coordinated_frames / coordinated_schedule / gather_frames
                    pinned: a hand-worked selection; first window = the pool in order;
                    later blocks distinct, disjoint from the previous block, in permutation
                    order; gathered rows equal the pool's frames
"""
from .dualparal import (as_f64, row_blocks, lookup, modulate, modulate_rounded,
                        window_attention, window_step, KVCacheRing, FifoQueue,
                        entry_step, long_run_schedule, timestep_schedule, LongRun)
from .sublayer import round_to, layer_norm, ln_modulate, linear, sublayer_step
from .noise_init import coordinated_frames, coordinated_schedule, gather_frames
from .context import fresh_context, fresh_context_sublayer

__all__ = ["as_f64", "row_blocks", "lookup", "modulate", "modulate_rounded",
           "window_attention", "window_step", "KVCacheRing", "FifoQueue", "entry_step",
           "long_run_schedule", "timestep_schedule", "LongRun", "round_to", "layer_norm",
           "ln_modulate", "linear", "sublayer_step", "coordinated_frames",
           "coordinated_schedule", "gather_frames", "fresh_context",
           "fresh_context_sublayer"]

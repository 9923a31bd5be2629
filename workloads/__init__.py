"""Seeded synthetic workloads for the DualParal window step.

This package holds only shapes and seeded random draws.  It contains none of
the method's arithmetic (no modulation, no attention, no queue logic), so both
the CPU oracle (``oracle/``) and the CUDA path (``long_video_diffusion_b200``)
can consume the same inputs without sharing any code that computes results.
"""
from .configs import (StepConfig, RunConfig, step_config, run_config, sweep_configs,
                      CONFIG_NAMES)
from .gen import (make_step_inputs, make_run_noise, make_run_table, to_dtype, as_features,
                  make_sublayer_weights, make_noise_permutations, make_run_pool)

__all__ = ["StepConfig", "RunConfig", "step_config", "run_config", "sweep_configs",
           "CONFIG_NAMES", "make_step_inputs", "make_run_noise", "make_run_table",
           "to_dtype", "as_features", "make_sublayer_weights",
           "make_noise_permutations", "make_run_pool"]

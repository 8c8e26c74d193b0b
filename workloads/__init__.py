"""Seeded synthetic input generators shared by the CUDA path's tests/bench and the CPU oracle.

Holds no verification arithmetic: only workload shapes, seeded random tensors and the
Philox4x32-10 uniform generator.
"""
from .configs import CONFIGS, StepConfig, sweep_config, SWEEP_LEVELS  # noqa: F401
from .philox import philox4x32, step_uniforms  # noqa: F401

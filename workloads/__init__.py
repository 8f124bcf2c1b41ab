"""Seeded synthetic inputs for the grouped NVFP4 MoE expert forward.

This package only draws inputs (weights, activations, routing).  It holds none
of the expert forward's arithmetic, so the CPU oracle and the CUDA path can
both consume its output without sharing any computation.
"""

from .generators import (  # noqa: F401
    CONFIGS,
    MATRIX_DOWN,
    MATRIX_GATE,
    MATRIX_UP,
    MoEProblem,
    make_problem,
)

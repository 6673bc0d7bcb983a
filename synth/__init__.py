"""Seeded synthetic inputs shared by the tests, the oracle checks and the benchmark.

This package holds no arithmetic of the method: it only draws per-turn
segment lengths, groups turns into conversations and sequences, and draws
Gaussian tensors.  The layout (duplication, position ids, masks) is computed
separately by the oracle and by the CUDA library.
"""

from .workloads import (  # noqa: F401
    CONFIGS,
    Workload,
    make_workload,
    make_custom_workload,
    npass_workload,
    random_small_workload,
    DEPTH_SWEEP_TURNS,
    gaussian,
    round_bf16,
)

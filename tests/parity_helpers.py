"""Shared pieces of the GPU parity tests: seeded inputs, error metrics, tolerances.

Float standard (bf16 inputs, fp32 accumulation): max |gpu - oracle| <= 1e-2 and
||gpu - oracle||_2 / ||oracle||_2 <= 5e-3 for O, LSE, dQ, dK and dV.
Layout outputs and the block map must match bit for bit.
"""

from __future__ import annotations

import numpy as np
import torch

MAX_ABS = 1e-2
REL_RMS = 5e-3


def errors(gpu, ref):
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    diff = g - r
    return float(np.abs(diff).max()), float(np.linalg.norm(diff) / max(np.linalg.norm(r), 1e-30))


def assert_close(name, gpu, ref, max_abs=MAX_ABS, rel_rms=REL_RMS):
    ma, rr = errors(gpu, ref)
    assert ma <= max_abs and rr <= rel_rms, f"{name}: max-abs {ma:.3e} (<= {max_abs}), rel-RMS {rr:.3e} (<= {rel_rms})"
    return ma, rr


def inputs(w, seed, with_do=True):
    """bf16-valued Q/K/V (and dO) ~ N(0, 1) for workload w, drawn from default_rng(seed)."""
    from synth import gaussian

    rng = np.random.default_rng(seed)
    total = w.total_tokens
    q = gaussian(rng, (total, w.hq, w.d))
    k = gaussian(rng, (total, w.hkv, w.d))
    v = gaussian(rng, (total, w.hkv, w.d))
    do = gaussian(rng, (total, w.hq, w.d)) if with_do else None
    return q, k, v, do


def to_dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(device="cuda", dtype=torch.bfloat16)

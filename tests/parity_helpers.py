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


def attention_order(lay) -> np.ndarray:
    """Stream index of each attention position (the order the attention calls take q, k and v
    in, include/opr.h attn_pos): per conversation its context tokens (h, r^in), then its trained
    tokens (t, r^out), each group in stream order.  Conversation ids grow along the stream, so
    one stable sort by (conversation, trained?) gives it; `lay` is an oracle layout."""
    from oracle import opr_oracle as orc

    idx = np.arange(len(lay.token_type))
    trained = (lay.token_type == orc.T) | (lay.token_type == orc.ROUT)
    return idx[np.lexsort((idx, trained.astype(np.int64), lay.conv_idx.astype(np.int64)))]


def block_map_in_order(lay, order, tile: int = 128) -> np.ndarray:
    """uint8 [n_seqs, T, T] block-map bytes (class | seen key halves << 2) of the oracle mask
    with rows and columns taken in `order` (stream index of each position)."""
    from oracle import opr_oracle as orc

    nt = (lay.max_seqlen + tile - 1) // tile
    out = np.zeros((lay.n_seqs, nt, nt), dtype=np.uint8)
    for s in range(lay.n_seqs):
        a, b = int(lay.cu_seqlens[s]), int(lay.cu_seqlens[s + 1])
        L = b - a
        perm = order[a:b]
        cnt = np.zeros((nt, nt, 2), dtype=np.int64)
        half_edges = np.arange(0, L, tile // 2)
        for qpos in range(L):
            row = orc.mask_row(lay, int(perm[qpos]), a, b)[perm - a].astype(np.int64)
            hs = np.add.reduceat(row, half_edges) if L else np.zeros(0, dtype=np.int64)
            hh = np.zeros(2 * nt, dtype=np.int64)
            hh[:len(hs)] = hs
            cnt[qpos // tile] += hh.reshape(nt, 2)
        tot = cnt.sum(axis=2)
        cls = np.where(tot == 0, orc.EMPTY, np.where(tot == tile * tile, orc.FULL, orc.PARTIAL))
        halves = (cnt[:, :, 0] > 0).astype(np.int64) | ((cnt[:, :, 1] > 0).astype(np.int64) << 1)
        out[s] = (cls | (halves << 2)).astype(np.uint8)
    return out

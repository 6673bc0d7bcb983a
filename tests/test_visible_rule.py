"""The visibility rule of the attention kernels and the layout (csrc/opr_internal.cuh,
visible(): same conversation, key not after query, the per-type rules of earlier and same
turns, later turns never), compiled for the host, against the oracle's mask ("分块稀疏注意力掩码")
for every (query, key) pair of small packed workloads, in the stream order and in the
attention order the kernels use (per conversation: context tokens, then trained tokens)."""

import os
import shutil
import subprocess

import numpy as np
import pytest

import synth
from oracle import opr_oracle as orc
from parity_helpers import attention_order

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.fixture(scope="module")
def rule_exe():
    if not os.path.exists(NVCC) and shutil.which("nvcc") is None:
        pytest.skip("needs nvcc")
    out_dir = os.path.join(ROOT, ".pytest_cache", "visible_rule")  # git-ignored
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "visible_rule")
    r = subprocess.run([NVCC if os.path.exists(NVCC) else "nvcc", "-std=c++17", "-o", exe,
                        os.path.join(ROOT, "tests", "c", "visible_rule.cu")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


@pytest.mark.parametrize("seed", range(3))
@pytest.mark.parametrize("order_name", ["stream", "attention"])
def test_visible_rule_matches_the_oracle_mask(rule_exe, seed, order_name):
    w = synth.random_small_workload(200 + seed, n_seqs=2, max_convs=3, max_turns=4)
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    order = attention_order(lay) if order_name == "attention" else np.arange(len(lay.token_type))
    conv = lay.conv_idx[order].astype(np.int64)
    meta = (lay.turn_idx[order].astype(np.int64) << 2) | lay.token_type[order].astype(np.int64)
    lines, ref = [], []
    for s in range(lay.n_seqs):
        a, b = int(lay.cu_seqlens[s]), int(lay.cu_seqlens[s + 1])
        perm = order[a:b] - a
        m = orc.dense_mask(lay, s)[np.ix_(perm, perm)]
        for qi in range(b - a):
            for ki in range(b - a):
                lines.append(f"{a + qi} {conv[a + qi]} {meta[a + qi]} {a + ki} {conv[a + ki]} {meta[a + ki]}")
                ref.append(int(m[qi, ki]))
    r = subprocess.run([rule_exe], input="\n".join(lines) + "\n", capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    got = np.array([int(x) for x in r.stdout.split()])
    ref = np.array(ref)
    assert got.shape == ref.shape
    assert int(ref.sum()) > 0
    np.testing.assert_array_equal(got, ref)

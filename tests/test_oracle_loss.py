"""Pins of the oracle's loss side (loss_rows, cross_entropy), without a GPU.

The pages prove that the one-pass loss equals the N-pass loss ("理论保证").
The pins: a hand-derived list of loss rows and targets for the worked example;
a two-layer toy transformer (RoPE attention under the one-pass mask, MLP,
residuals) whose one-pass losses equal those of the N-pass runs to 1e-10;
cross-entropy against its closed forms and PyTorch's float64 routine.
"""

import os

import numpy as np
import pytest
import torch

import synth
from oracle import opr_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example_two_turns_loss_rows.txt")


def test_worked_example_loss_rows():
    rows, targets = orc.loss_rows([[2, 3, 2], [1, 2, 1]], [0, 2])
    g = [tuple(int(x) for x in line.split()[1:]) for line in open(GOLDEN) if line.startswith("row ")]
    assert list(zip(rows.tolist(), targets.tolist())) == g


def test_loss_rows_are_last_h_t_and_r_out_rows():
    w = synth.random_small_workload(3, max_turns=5)
    rows, targets = orc.loss_rows(w.turn_lens, w.conv_turn_ptr)
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    types = lay.token_type[rows]
    assert set(types.tolist()) <= {orc.H, orc.T, orc.ROUT}
    # every t row and every r^out row but the last of its turn carries a loss
    lens = np.asarray(w.turn_lens).reshape(-1, 3)
    n_expected = sum((1 if h > 0 and t + r > 0 else 0) + (t if r > 0 else max(t - 1, 0)) + max(r - 1, 0)
                     for h, t, r in lens)
    assert len(rows) == n_expected
    assert np.all(np.diff(rows) > 0)


class ToyModel:
    """Two pre-norm-free transformer layers (RoPE attention with GQA, ReLU MLP, residuals)
    and a linear head, float64, random weights."""

    def __init__(self, V=37, dm=16, hq=2, hkv=1, d=8, seed=0):
        rng = np.random.default_rng(seed)
        g = lambda *s: rng.standard_normal(s) / np.sqrt(s[0])  # noqa: E731
        self.V, self.hq, self.hkv, self.d = V, hq, hkv, d
        self.E = rng.standard_normal((V, dm))
        self.layers = [dict(q=g(dm, hq * d), k=g(dm, hkv * d), v=g(dm, hkv * d), o=g(hq * d, dm),
                            w1=g(dm, 2 * dm), w2=g(2 * dm, dm)) for _ in range(2)]
        self.out = g(dm, V)

    def logits(self, ids, attend):
        x = self.E[ids]
        n = len(ids)
        for L in self.layers:
            q = (x @ L["q"]).reshape(n, self.hq, self.d)
            k = (x @ L["k"]).reshape(n, self.hkv, self.d)
            v = (x @ L["v"]).reshape(n, self.hkv, self.d)
            x = x + attend(q, k, v).reshape(n, -1) @ L["o"]
            x = x + np.maximum(x @ L["w1"], 0.0) @ L["w2"]
        return x @ self.out


@pytest.mark.parametrize("seed", [0, 1])
def test_toy_model_one_pass_loss_equals_n_pass(seed):
    w = synth.random_small_workload(seed, n_seqs=1, max_convs=2, max_turns=4, h=(0, 9), t=(0, 9), r=(0, 9))
    rng = np.random.default_rng(seed + 10)
    model = ToyModel(seed=seed)
    lens = np.asarray(w.turn_lens).reshape(-1, 3)
    ids = rng.integers(0, model.V, size=int(lens.sum()))
    base = 1e4
    # one pass
    src, _ = orc.duplication_index(w.turn_lens, w.conv_turn_ptr)
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    z = model.logits(ids[src], lambda q, k, v: orc.forward(q, k, v, lay, base)[0])
    rows, targets = orc.loss_rows(w.turn_lens, w.conv_turn_ptr)
    one_pass, _ = orc.cross_entropy(z[rows], ids[targets])
    # N pass: one causal run per turn over [H<i, h_i, t_i, r_i], contiguous positions
    npass = []
    orig = 0
    for c in range(len(w.conv_turn_ptr) - 1):
        hist = []
        for t in range(w.conv_turn_ptr[c], w.conv_turn_ptr[c + 1]):
            h, tt, r = (int(x) for x in lens[t])
            seq = hist + list(range(orig, orig + h + tt + r))
            n = len(seq)
            pos = np.arange(n)
            zz = model.logits(ids[seq], lambda q, k, v: orc.causal_attention(orc.rope(q, pos, base),
                                                                             orc.rope(k, pos, base), v)[0])
            start = len(hist)
            for p in range(start + h - 1 if h > 0 else start + h, n - 1):
                if p >= start + h - 1 and p >= 0 and seq[p + 1] >= orig + h:
                    l, _ = orc.cross_entropy(zz[p:p + 1], ids[[seq[p + 1]]])
                    npass.append(l[0])
            hist += list(range(orig, orig + h)) + list(range(orig + h + tt, orig + h + tt + r))
            orig += h + tt + r
    np.testing.assert_allclose(one_pass, np.asarray(npass), rtol=0, atol=1e-10)


def test_cross_entropy_closed_forms_and_torch():
    rng = np.random.default_rng(0)
    z = rng.standard_normal((7, 11)) * 3
    tgt = rng.integers(0, 11, size=7)
    loss, dz = orc.cross_entropy(z, tgt)
    zt = torch.tensor(z, requires_grad=True)
    lt = torch.nn.functional.cross_entropy(zt, torch.tensor(tgt), reduction="sum")
    lt.backward()
    np.testing.assert_allclose(loss.sum(), lt.item(), rtol=1e-13)
    np.testing.assert_allclose(dz, zt.grad.numpy(), atol=1e-13)
    u, du = orc.cross_entropy(np.zeros((2, 5)), [0, 3])
    np.testing.assert_allclose(u, np.log(5.0))
    np.testing.assert_allclose(du.sum(axis=1), 0.0, atol=1e-15)

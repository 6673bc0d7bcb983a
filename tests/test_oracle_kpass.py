"""Pins of the oracle's K-pass arrangement (kpass_plan, kpass_index) without a GPU.

K-pass sits between N-pass (K = N) and one-pass (K = 1) ("K-Pass 中间方案"):
each pass is a group of turns behind the history of the earlier turns (h_j
and r_j as context).  The pins: K = 1 is the one-pass layout; every copy of a
token has the forward row that Theorem 2.1 gives it in one pass (context
copies the h / r^in row, the r^out copy the r^out row), for K = 2 and K = N;
copy counts per token type; the fold as the adjoint of the gather.
"""

import numpy as np
import pytest

import synth
from oracle import opr_oracle as orc

TURNS = [[[2, 3, 2], [1, 2, 1], [3, 1, 2], [0, 2, 1]], [[4, 2, 3], [2, 0, 2]]]  # two conversations


def _flat(convs):
    lens = [t for c in convs for t in c]
    ptr = np.cumsum([0] + [len(c) for c in convs])
    return np.asarray(lens, dtype=np.int32), ptr.astype(np.int32)


def test_k1_is_the_one_pass_layout():
    lens, ptr = _flat(TURNS)
    l2, c2, s2, tsrc = orc.kpass_plan(lens, ptr, [0, len(TURNS)], 1)
    np.testing.assert_array_equal(l2, lens.reshape(-1, 3))
    np.testing.assert_array_equal(c2, ptr)
    src, copies = orc.kpass_index(lens, ptr, [0, len(TURNS)], 1)
    d_src, d_copies = orc.duplication_index(lens, ptr)
    np.testing.assert_array_equal(src, d_src)
    np.testing.assert_array_equal(copies, d_copies)


@pytest.mark.parametrize("K", [2, 3, 4])
def test_copy_counts(K):
    lens, ptr = _flat(TURNS)
    src, copies = orc.kpass_index(lens, ptr, [0, len(TURNS)], K)
    n_copies = (copies >= 0).sum(axis=1)
    np.testing.assert_array_equal(np.bincount(src, minlength=len(copies)), n_copies)
    o = 0
    for conv in TURNS:
        b = orc.kpass_groups(len(conv), K)
        for j, (h, t, r) in enumerate(conv):
            g = next(q for q in range(len(b) - 1) if b[q] <= j < b[q + 1])
            later = len(b) - 2 - g
            assert list(n_copies[o:o + h]) == [1 + later] * h
            assert list(n_copies[o + h:o + h + t]) == [1] * t
            assert list(n_copies[o + h + t:o + h + t + r]) == [2 + later] * r
            o += h + t + r
    for i, oi in enumerate(src):
        assert i in copies[oi]


@pytest.mark.parametrize("K", [2, 4])
def test_every_copy_has_its_one_pass_row(K):
    """Theorem 2.1 through the K-pass arrangement: O and LSE rows of each copy equal the one-pass row
    of that token (context copies the h / r^in row, r^out copies the r^out row) to 1e-12."""
    lens, ptr = _flat(TURNS)
    seqs = [0, len(TURNS)]
    rng = np.random.default_rng(0)
    n_orig = int(lens.sum())
    hq, hkv, d, base = 2, 1, 16, 1e4
    q0 = rng.standard_normal((n_orig, hq, d))
    k0 = rng.standard_normal((n_orig, hkv, d))
    v0 = rng.standard_normal((n_orig, hkv, d))
    d_src, d_copies = orc.duplication_index(lens, ptr)
    lay1 = orc.build_layout(lens, ptr, seqs)
    o1, lse1 = orc.forward(q0[d_src], k0[d_src], v0[d_src], lay1, base)
    l2, c2, s2, _ = orc.kpass_plan(lens, ptr, seqs, K)
    k_src, k_copies = orc.kpass_index(lens, ptr, seqs, K)
    layk = orc.build_layout(l2, c2, s2)
    ok, lsek = orc.forward(q0[k_src], k0[k_src], v0[k_src], layk, base)
    for o in range(n_orig):
        for slot, pos in enumerate(k_copies[o]):
            if pos < 0:
                continue
            ref = d_copies[o, 1] if slot == 1 else d_copies[o, 0]
            np.testing.assert_allclose(ok[pos], o1[ref], rtol=0, atol=1e-12)
            np.testing.assert_allclose(lsek[:, pos], lse1[:, ref], rtol=0, atol=1e-12)


def test_planted_history_order_is_caught():
    """History segments fed r_j before h_j (a plausible slip) change the later rows: the row pin fails."""
    lens, ptr = _flat(TURNS)
    seqs = [0, len(TURNS)]
    rng = np.random.default_rng(2)
    n_orig = int(lens.sum())
    q0, k0, v0 = (rng.standard_normal((n_orig, 1, 16)) for _ in range(3))
    d_src, d_copies = orc.duplication_index(lens, ptr)
    o1, _ = orc.forward(q0[d_src], k0[d_src], v0[d_src], orc.build_layout(lens, ptr, seqs), 1e4)
    l2, c2, s2, tsrc = orc.kpass_plan(lens, ptr, seqs, 2)
    k_src, k_copies = orc.kpass_index(lens, ptr, seqs, 2)
    bad_src = k_src.copy()
    pos = 0
    for (n, t, r), (j, dd) in zip(l2, tsrc):  # noqa: B007
        n_tok = int(n) + int(t) + 2 * int(r)
        if dd >= 1:
            h_j = int(lens[j][0])
            seg = bad_src[pos:pos + n_tok].copy()
            bad_src[pos:pos + n_tok] = np.concatenate([seg[h_j:], seg[:h_j]])  # r_j first
        pos += n_tok
    ok_bad, _ = orc.forward(q0[bad_src], k0[bad_src], v0[bad_src], orc.build_layout(l2, c2, s2), 1e4)
    worst = 0.0
    for o in range(n_orig):
        for slot, p in enumerate(k_copies[o]):
            if p >= 0:
                ref = d_copies[o, 1] if slot == 1 else d_copies[o, 0]
                worst = max(worst, float(np.abs(ok_bad[p] - o1[ref]).max()))
    assert worst > 1e-3


def test_fold_is_the_adjoint_of_gather():
    w = synth.random_small_workload(9, max_turns=5)
    src, copies = orc.kpass_index(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, 3)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((len(copies), 5))
    dy = rng.standard_normal((len(src), 5)).astype(np.float32)
    lhs = float(np.sum(orc.gather_rows(x, src) * dy.astype(np.float64)))
    rhs = float(np.sum(x * orc.fold_rows(dy, copies).astype(np.float64)))
    assert abs(lhs - rhs) <= 1e-5 * (abs(lhs) + 1.0)

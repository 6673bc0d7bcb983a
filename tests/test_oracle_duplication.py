"""Pins of the oracle's token-duplication step (duplication_index, gather_rows,
fold_rows) against the pages and plain counting, without a GPU.

The one-pass stream stores every response twice (r^in and r^out) after h and
t ("Token 复制" in the One-Pass to Reason wiki note).  The pins: a hand-derived
map of the worked example, closed-form stream lengths, the copy structure
(each h / t token once, each r token twice, both copies of a turn's r in
order), consistency with the layout's token types, and the fold as the exact
adjoint of the gather.
"""

import os

import numpy as np
import pytest

import synth
from oracle import opr_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example_two_turns_duplication.txt")


def _golden():
    src, copies = None, []
    for line in open(GOLDEN):
        f = line.split()
        if not f or f[0].startswith("#"):
            continue
        if f[0] == "src":
            src = [int(x) for x in f[1:]]
        elif f[0] == "copy":
            copies.append([int(f[1]), int(f[2])])
    return np.asarray(src), np.asarray(copies)


def test_worked_example_matches_hand_derived_map():
    src, copies = orc.duplication_index([[2, 3, 2], [1, 2, 1]], [0, 2])
    g_src, g_copies = _golden()
    np.testing.assert_array_equal(src, g_src)
    np.testing.assert_array_equal(copies, g_copies)


def _structure_checks(w):
    src, copies = orc.duplication_index(w.turn_lens, w.conv_turn_ptr)
    lens = np.asarray(w.turn_lens).reshape(-1, 3)
    h, t, r = lens[:, 0].sum(), lens[:, 1].sum(), lens[:, 2].sum()
    assert len(src) == h + t + 2 * r == w.total_tokens
    assert len(copies) == h + t + r
    # every original token appears once, r tokens twice; copies is the inverse of src
    counts = np.bincount(src, minlength=len(copies))
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    for o, (a, b) in enumerate(copies):
        assert src[a] == o
        if b >= 0:
            assert src[b] == o and counts[o] == 2
            assert lay.token_type[a] == orc.RIN and lay.token_type[b] == orc.ROUT
            # both copies of a turn's r in the same order: the same offset into r_in and r_out
            assert b - a == _r_len(lay, a)
        else:
            assert counts[o] == 1 and lay.token_type[a] in (orc.H, orc.T)
    # the original stream is the one-pass stream without the r^out tokens, in order
    keep = lay.token_type != orc.ROUT
    np.testing.assert_array_equal(src[keep], np.arange(len(copies)))


def _r_len(lay, a):
    """Length of the r^in run containing token a (its r^out copy starts that far on)."""
    e = a
    while e < lay.total and lay.token_type[e] == orc.RIN and lay.turn_idx[e] == lay.turn_idx[a]:
        e += 1
    s = a
    while s > 0 and lay.token_type[s - 1] == orc.RIN and lay.turn_idx[s - 1] == lay.turn_idx[a]:
        s -= 1
    return e - s


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_structure_on_random_workloads(seed):
    _structure_checks(synth.random_small_workload(seed))


def test_structure_with_zero_length_segments():
    w = synth.make_custom_workload([[[[0, 3, 2], [2, 0, 0], [1, 1, 0], [0, 0, 3]]], [[[4, 0, 1]]]],
                                   hq=1, hkv=1, d=64, base=1e4)
    _structure_checks(w)


def test_fold_is_the_adjoint_of_gather():
    """<gather(x), dy> = <x, fold(dy)> for random x and dy: fold is the exact transpose."""
    w = synth.random_small_workload(5)
    src, copies = orc.duplication_index(w.turn_lens, w.conv_turn_ptr)
    rng = np.random.default_rng(0)
    x = rng.standard_normal((len(copies), 6))
    dy = rng.standard_normal((len(src), 6)).astype(np.float32)
    lhs = float(np.sum(orc.gather_rows(x, src) * dy.astype(np.float64)))
    rhs = float(np.sum(x * orc.fold_rows(dy, copies).astype(np.float64)))
    assert abs(lhs - rhs) <= 1e-5 * (abs(lhs) + 1.0)


def test_fold_of_gather_counts_copies():
    """fold(gather(x)) = x times the number of copies (1 for h and t, 2 for r)."""
    src, copies = orc.duplication_index([[2, 3, 2], [1, 2, 1]], [0, 2])
    x = np.arange(len(copies), dtype=np.float32)[:, None] + 1.0
    got = orc.fold_rows(orc.gather_rows(x, src), copies)
    mult = np.where(copies[:, 1] >= 0, 2.0, 1.0)[:, None]
    np.testing.assert_array_equal(got, x * mult)


def test_planted_swap_of_rin_and_rout_is_caught():
    """A map whose r^out copies point at the next original token fails the worked example."""
    src, copies = orc.duplication_index([[2, 3, 2], [1, 2, 1]], [0, 2])
    bad = src.copy()
    bad[7], bad[8] = bad[8], bad[7]
    g_src, _ = _golden()
    assert not np.array_equal(bad, g_src)

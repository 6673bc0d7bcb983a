"""Property tests of the oracle's token maps over arbitrary turn lengths (hypothesis):
zero-length segments, one-turn conversations, many conversations."""

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import opr_oracle as orc

turn = st.tuples(st.integers(0, 5), st.integers(0, 5), st.integers(0, 5))
convs = st.lists(st.lists(turn, min_size=1, max_size=5), min_size=1, max_size=4)


def _flat(cs):
    lens = np.asarray([t for c in cs for t in c], dtype=np.int32).reshape(-1, 3)
    ptr = np.cumsum([0] + [len(c) for c in cs]).astype(np.int32)
    return lens, ptr


@settings(max_examples=60, deadline=None)
@given(convs)
def test_duplication_map_is_a_consistent_copy(cs):
    lens, ptr = _flat(cs)
    src, copies = orc.duplication_index(lens, ptr)
    assert len(src) == int(lens[:, 0].sum() + lens[:, 1].sum() + 2 * lens[:, 2].sum())
    assert len(copies) == int(lens.sum())
    for o, (a, b) in enumerate(copies):
        assert src[a] == o and (b < 0 or src[b] == o)
    assert np.array_equal(np.bincount(src, minlength=len(copies)), (copies >= 0).sum(axis=1))


@settings(max_examples=40, deadline=None)
@given(convs, st.integers(1, 6))
def test_kpass_map_is_a_consistent_copy(cs, K):
    lens, ptr = _flat(cs)
    seqs = [0, len(cs)]
    l2, c2, s2, tsrc = orc.kpass_plan(lens, ptr, seqs, K)
    src, copies = orc.kpass_index(lens, ptr, seqs, K)
    assert len(src) == int(l2[:, 0].sum() + l2[:, 1].sum() + 2 * l2[:, 2].sum())
    for o, row in enumerate(copies):
        assert row[0] >= 0  # every original token has its own-pass copy
        for p in row:
            assert p < 0 or src[p] == o
    # every loss-carrying turn appears exactly once as an own-group turn
    own = tsrc[tsrc[:, 1] < 0, 0]
    assert np.array_equal(np.sort(own), np.arange(len(lens)))


@settings(max_examples=60, deadline=None)
@given(convs)
def test_loss_rows_targets_are_the_next_assistant_token(cs):
    lens, ptr = _flat(cs)
    rows, targets = orc.loss_rows(lens, ptr)
    src, _ = orc.duplication_index(lens, ptr)
    lay = orc.build_layout(lens, ptr, [0, len(cs)])
    assert np.all(np.diff(rows) > 0)
    for r_, t_ in zip(rows, targets):
        # the target is an assistant (t or r) token right after the row's own original token,
        # except from the last h row, whose target follows the h segment
        assert lay.token_type[r_] in (orc.H, orc.T, orc.ROUT)
        assert t_ == src[r_] + 1

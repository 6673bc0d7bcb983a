"""Pins of the oracle's layout, mask and block map (no GPU).

Each check is computed here from the pages' statements by a route other than
the oracle's own code: the hand-derived worked example, the position-id
formulas applied to segment ends, closed-form pair counts per turn, and a
double-loop tile count.
"""

import os

import numpy as np
import pytest

import synth
from oracle import opr_oracle as orc

TYPES = {"h": orc.H, "t": orc.T, "rin": orc.RIN, "rout": orc.ROUT}


def load_golden(path):
    toks, rows, npass = [], [], None
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        f = line.split()
        if f[0] == "turns":
            turns = np.array([int(x) for x in f[1:]], dtype=np.int32).reshape(-1, 3)
        elif f[0] == "tok":
            toks.append((int(f[1]), TYPES[f[2]], int(f[3]), int(f[4])))
        elif f[0] == "row":
            rows.append([c == "1" for c in f[1]])
        elif f[0] == "npass1":
            npass = [int(x) for x in f[1:]]
    return turns, toks, np.array(rows, dtype=bool), npass


def test_worked_example(golden_dir):
    """Positions and visibility of a two-turn conversation, derived by hand."""
    turns, toks, rows, npass = load_golden(os.path.join(golden_dir, "worked_example_two_turns.txt"))
    lay = orc.build_layout(turns, [0, len(turns)], [0, 1])
    assert lay.total == len(toks)
    for idx, typ, turn, pos in toks:
        assert lay.token_type[idx] == typ
        assert lay.turn_idx[idx] == turn
        assert lay.pos_id[idx] == pos
    np.testing.assert_array_equal(orc.dense_mask(lay, 0), rows)
    # the N-pass sequence of turn 1 reuses exactly these one-pass tokens
    lists = orc.npass_token_lists(lay, turns, [0, len(turns)])
    assert list(lists[1][2]) == npass
    assert list(lay.pos_id[npass]) == list(range(len(npass)))


def _segments(lay):
    """(conv, turn, type) -> (first, last) token index, for non-empty segments."""
    seg = {}
    for i in range(lay.total):
        key = (int(lay.conv_idx[i]), int(lay.turn_idx[i]), int(lay.token_type[i]))
        a, _ = seg.get(key, (i, i))
        seg[key] = (a, i)
    return seg


@pytest.mark.parametrize("seed", range(6))
def test_position_formulas(seed):
    """s_t = s_rin = e_h + 1, s_rout = e_t + 1, s_h(i+1) = e_rin + 1; first position 0."""
    w = synth.random_small_workload(seed, h=(1, 40), t=(1, 60), r=(1, 40))
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    seg = _segments(lay)
    P = lay.pos_id
    for (c, i, typ), (a, b) in seg.items():
        assert np.all(np.diff(P[a:b + 1]) == 1), "positions contiguous inside a segment"
    for (c, i, typ), (a, b) in seg.items():
        if typ == orc.H:
            e_h = P[b]
            assert P[seg[(c, i, orc.T)][0]] == e_h + 1
            assert P[seg[(c, i, orc.RIN)][0]] == e_h + 1
            e_t = P[seg[(c, i, orc.T)][1]]
            assert P[seg[(c, i, orc.ROUT)][0]] == e_t + 1
            if (c, i + 1, orc.H) in seg:
                e_rin = P[seg[(c, i, orc.RIN)][1]]
                assert P[seg[(c, i + 1, orc.H)][0]] == e_rin + 1
            if i == 0:
                assert P[a] == 0
    # duplication: L = sum(h + t + 2r)
    assert lay.total == int((w.turn_lens[:, 0] + w.turn_lens[:, 1] + 2 * w.turn_lens[:, 2]).sum())
    np.testing.assert_array_equal(np.diff(lay.cu_seqlens), w.seq_lengths())


def _closed_form_pairs(turns):
    """Visible pairs per turn and type from the rules, with A_i = sum_{j<i}(h_j + r_j)."""
    out, A = [], 0
    for h, t, r in turns:
        h, t, r = int(h), int(t), int(r)
        out.append({
            orc.H: h * A + h * (h + 1) // 2,
            orc.T: t * (A + h) + t * (t + 1) // 2,
            orc.RIN: r * (A + h) + r * (r + 1) // 2,
            orc.ROUT: r * (A + h + t) + r * (r + 1) // 2,
        })
        A += h + r
    return out


@pytest.mark.parametrize("seed", range(8))
def test_pair_counts_closed_form(seed):
    w = synth.random_small_workload(seed)
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    for s in range(lay.n_seqs):
        a = int(lay.cu_seqlens[s])
        m = orc.dense_mask(lay, s)
        for c in range(w.seq_conv_ptr[s], w.seq_conv_ptr[s + 1]):
            t0, t1 = w.conv_turn_ptr[c], w.conv_turn_ptr[c + 1]
            expect = _closed_form_pairs(w.turn_lens[t0:t1])
            for i in range(t1 - t0):
                for typ in range(4):
                    rows = np.nonzero((lay.conv_idx[a:a + len(m)] == c) & (lay.turn_idx[a:a + len(m)] == i)
                                      & (lay.token_type[a:a + len(m)] == typ))[0]
                    assert int(m[rows].sum()) == expect[i][typ], (seed, c, i, typ)


@pytest.mark.parametrize("seed", range(6))
def test_mask_invariants(seed):
    """Subset of causal, diagonal always set, no visibility across conversations."""
    w = synth.random_small_workload(seed + 100)
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    for s in range(lay.n_seqs):
        a, b = int(lay.cu_seqlens[s]), int(lay.cu_seqlens[s + 1])
        m = orc.dense_mask(lay, s)
        assert not np.any(m & ~np.tril(np.ones_like(m)))
        assert np.all(np.diag(m))
        cv = lay.conv_idx[a:b]
        assert not np.any(m & (cv[:, None] != cv[None, :]))


def test_single_segment_is_causal():
    """One turn (n, 0, 0): the mask is the textbook causal mask."""
    lay = orc.build_layout([[37, 0, 0]], [0, 1], [0, 1])
    np.testing.assert_array_equal(orc.dense_mask(lay, 0), np.tril(np.ones((37, 37), dtype=bool)))
    np.testing.assert_array_equal(lay.pos_id, np.arange(37))


def test_zero_length_segments():
    """Empty t and r: positions continue from h; r_out with t = 0 starts after h."""
    lay = orc.build_layout([[3, 0, 2], [0, 2, 0], [1, 0, 0]], [0, 3], [0, 1])
    assert list(lay.token_type) == [0, 0, 0, 2, 2, 3, 3, 1, 1, 0]
    assert list(lay.pos_id) == [0, 1, 2, 3, 4, 3, 4, 5, 6, 5]


@pytest.mark.parametrize("tile", [4, 8, 16])
def test_block_map_bruteforce(tile):
    """Tile classes against a plain double loop over the dense mask."""
    w = synth.random_small_workload(7, h=(0, 20), t=(0, 30), r=(0, 20))
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    bm = orc.block_map(lay, tile=tile)
    nt = bm.shape[1]
    for s in range(lay.n_seqs):
        m = orc.dense_mask(lay, s)
        L = len(m)
        for I in range(nt):
            for J in range(nt):
                cnt = 0
                for qq in range(I * tile, (I + 1) * tile):
                    for kk in range(J * tile, (J + 1) * tile):
                        if qq < L and kk < L and m[qq, kk]:
                            cnt += 1
                want = 0 if cnt == 0 else (1 if cnt == tile * tile else 2)
                assert bm[s, I, J] == want


def test_visible_pairs_matches_closed_form():
    w = synth.make_workload(3, n_turns=2)
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    expect = sum(sum(d.values()) for d in _closed_form_pairs(w.turn_lens))
    # by hand: turn 0 gives 8256 + 196864 + 65664 + 196736, turn 1 (A = 384)
    # gives 57408 + 393472 + 163968 + 295040
    assert orc.visible_pairs(lay) == expect == 1377408


def test_key_half_map_by_brute_force():
    """key_half_map against the dense mask, and consistent with the block map (a tile is empty
    exactly when neither half is seen; a full tile has both halves seen)."""
    w = synth.random_small_workload(8, n_seqs=2, max_convs=3, max_turns=4)
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    km = orc.key_half_map(lay)
    bm = orc.block_map(lay)
    T = km.shape[1]
    for s in range(lay.n_seqs):
        m = orc.dense_mask(lay, s)
        L = m.shape[0]
        for I in range(T):
            for J in range(T):
                q = m[I * 128:min((I + 1) * 128, L)]
                bits = 0
                for h in range(2):
                    ks = slice(J * 128 + 64 * h, min(J * 128 + 64 * (h + 1), L))
                    if q.size and q[:, ks].size and q[:, ks].any():
                        bits |= 1 << h
                assert km[s, I, J] == bits
                assert (bits == 0) == (bm[s, I, J] == orc.EMPTY)
                if bm[s, I, J] == orc.FULL:
                    assert bits == 3


def test_key_half_map_of_a_causal_segment():
    """One causal segment of 256 tokens: the diagonal tiles see both key halves, the tile above
    the diagonal neither (closed form of the causal mask)."""
    lay = orc.build_layout([[256, 0, 0]], [0, 1], [0, 1])
    km = orc.key_half_map(lay)
    assert km[0].tolist() == [[3, 0], [3, 3]]


@pytest.mark.parametrize("seed", range(4))
def test_attention_order_keeps_every_visible_key_before_its_query(seed):
    """The attention kernels take tokens in the attention order (per conversation: context h,
    r^in, then trained t, r^out) and rely on "key not after query" there too: the mask with rows
    and columns in that order must stay lower triangular, each segment in stream order."""
    from parity_helpers import attention_order

    w = synth.random_small_workload(100 + seed, n_seqs=2, max_convs=3, max_turns=5)
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    order = attention_order(lay)
    assert sorted(order.tolist()) == list(range(len(order)))
    for s in range(lay.n_seqs):
        a, b = int(lay.cu_seqlens[s]), int(lay.cu_seqlens[s + 1])
        perm = order[a:b]
        assert perm.min() >= a and perm.max() < b  # a permutation inside the sequence
        m = orc.dense_mask(lay, s)[np.ix_(perm - a, perm - a)]
        assert not np.triu(m, 1).any()
        # inside a conversation: every context token before every trained token
        ty = lay.token_type[perm]
        cv = lay.conv_idx[perm]
        for c in np.unique(cv):
            t = ty[cv == c]
            trained = (t == orc.T) | (t == orc.ROUT)
            assert not (trained[:-1] & ~trained[1:]).any()


def test_block_map_in_order_reduces_to_the_oracle_block_map():
    """The test helper that builds the attention-order block map gives the oracle's block map
    and key-half map for the identity order."""
    from parity_helpers import block_map_in_order

    w = synth.random_small_workload(7, n_seqs=2, max_convs=3, max_turns=4)
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    got = block_map_in_order(lay, np.arange(len(lay.token_type)))
    np.testing.assert_array_equal(got & 3, orc.block_map(lay))
    np.testing.assert_array_equal(got >> 2, orc.key_half_map(lay))

"""Pins of the oracle's RoPE, attention and gradients (no GPU).

* Theorem 2.1 of One-Pass to Reason ("理论保证"; English note, "Method" item 4)
  by brute force: one causal run per turn over [h_1 r_1 ... h_i t_i r_i] with
  contiguous positions must give the same rows as the one-pass layout, to 1e-12.
* The single-segment case equals PyTorch's float64 causal
  scaled_dot_product_attention, an independent library routine.
* RoPE: norm preserved, q(m).k(n) depends only on m - n, position 0 is the
  identity, d = 2 is a plane rotation.
* Gradients: central finite differences of <dO, O> in float64.
* Planted mistakes in the oracle's mask are caught by the Theorem check.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import opr_oracle as orc


def _inputs(w, rng, fp32=True):
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    n = lay.total
    q = rng.standard_normal((n, w.hq, w.d))
    k = rng.standard_normal((n, w.hkv, w.d))
    v = rng.standard_normal((n, w.hkv, w.d))
    return lay, q, k, v


def _theorem_max_err(w, rng):
    lay, q, k, v = _inputs(w, rng)
    o, lse = orc.forward(q, k, v, lay, w.base)
    err = 0.0
    for c, i, toks, on, lsen in orc.npass_rows(q, k, v, lay, w.turn_lens, w.conv_turn_ptr, w.base):
        # every row of the N-pass run: history h_j / r_j^in, and h_i, t_i, r_i^out
        err = max(err, np.abs(o[toks] - on).max(), np.abs(lse[:, toks] - lsen).max())
    return err


@pytest.mark.parametrize("seed", range(5))
def test_theorem_2_1_one_pass_equals_n_pass(seed):
    w = synth.random_small_workload(seed, n_seqs=2, max_convs=2, max_turns=4,
                                    h=(1, 12), t=(0, 20), r=(0, 12), hq=4, hkv=2, d=16, base=1e4)
    assert _theorem_max_err(w, np.random.default_rng(seed)) < 1e-12


def test_theorem_2_1_tiny_config():
    """The tiny workload (N = 2, h16 t32 r16, d 64, RoPE base 1e4)."""
    w = synth.make_workload(0)
    assert _theorem_max_err(w, np.random.default_rng(1000)) < 1e-12


PLANTED = {
    "r_out sees r_in of its turn": lambda ty, tau, cur: (tau == orc.ROUT) & cur & (ty == orc.RIN),
    "r_in sees t of its turn": lambda ty, tau, cur: (tau == orc.RIN) & cur & (ty == orc.T),
    "history includes t": lambda ty, tau, cur: ~cur & (ty == orc.T),
    "history includes r_out": lambda ty, tau, cur: ~cur & (ty == orc.ROUT),
}


@pytest.mark.parametrize("name", sorted(PLANTED))
def test_planted_mask_mistakes_are_caught(monkeypatch, name):
    """A wrong visibility rule planted in the oracle breaks the Theorem check."""
    extra = PLANTED[name]
    real = orc.mask_row

    def wrong(lay, q, lo, hi):
        row = real(lay, q, lo, hi)
        idx = np.arange(lo, hi)
        ty, tu, cv = lay.token_type[lo:hi], lay.turn_idx[lo:hi], lay.conv_idx[lo:hi]
        same = (cv == lay.conv_idx[q]) & (idx <= q)
        cur = tu == lay.turn_idx[q]
        return row | (same & extra(ty, lay.token_type[q], cur))

    monkeypatch.setattr(orc, "mask_row", wrong)
    w = synth.make_custom_workload([[[(3, 4, 3), (2, 5, 2), (4, 3, 3)]]], hq=2, hkv=1, d=8)
    assert _theorem_max_err(w, np.random.default_rng(5)) > 1e-3


def test_planted_position_mistake_is_caught(monkeypatch):
    """r_out placed after r_in instead of after t breaks the Theorem check."""
    real = orc.build_layout

    def wrong(*a):
        lay = real(*a)
        pos = lay.pos_id.copy()
        rout = lay.token_type == orc.ROUT
        pos[rout] += 1
        lay.pos_id = pos
        return lay

    monkeypatch.setattr(orc, "build_layout", wrong)
    w = synth.make_custom_workload([[[(3, 4, 3), (2, 5, 2)]]], hq=2, hkv=1, d=8)
    assert _theorem_max_err(w, np.random.default_rng(6)) > 1e-6


def test_single_segment_matches_torch_sdpa():
    rng = np.random.default_rng(3)
    w = synth.make_custom_workload([[[(45, 0, 0)]], [[(30, 0, 0)]]], hq=4, hkv=2, d=32, base=1e4)
    lay, q, k, v = _inputs(w, rng)
    o, lse = orc.attention_fwd(q, k, v, lay)
    for s in range(lay.n_seqs):
        a, b = int(lay.cu_seqlens[s]), int(lay.cu_seqlens[s + 1])
        qt = torch.from_numpy(q[a:b]).permute(1, 0, 2)
        kt = torch.from_numpy(k[a:b]).permute(1, 0, 2).repeat_interleave(2, dim=0)
        vt = torch.from_numpy(v[a:b]).permute(1, 0, 2).repeat_interleave(2, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
        np.testing.assert_allclose(o[a:b], ref.permute(1, 0, 2).numpy(), atol=1e-12, rtol=0)
        # LSE: log of the softmax denominator, from the raw scores
        sc = (qt @ kt.transpose(1, 2)).numpy() / np.sqrt(32)
        sc = np.where(np.tril(np.ones((b - a, b - a), dtype=bool)), sc, -np.inf)
        ref_lse = np.log(np.exp(sc).sum(-1))
        np.testing.assert_allclose(lse[:, a:b], ref_lse, atol=1e-12, rtol=0)


def test_rope_invariants():
    rng = np.random.default_rng(0)
    d = 64
    x = rng.standard_normal((50, 3, d))
    pos = rng.integers(0, 100000, size=50)
    y = orc.rope(x, pos, 1e6)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    np.testing.assert_allclose(orc.rope(y, pos, 1e6, inverse=True), x, atol=1e-12)
    np.testing.assert_array_equal(orc.rope(x, np.zeros(50, dtype=int), 1e6), x)
    # relative position: <R(m) a, R(n) b> depends on m - n only
    a, b = rng.standard_normal((1, 1, d)), rng.standard_normal((1, 1, d))
    ref = (orc.rope(a, [7], 1e4) * orc.rope(b, [3], 1e4)).sum()
    for shift in (1, 100, 12345):
        got = (orc.rope(a, [7 + shift], 1e4) * orc.rope(b, [3 + shift], 1e4)).sum()
        assert abs(got - ref) < 1e-10
    # d = 2: a plane rotation by pos radians (theta_0 = 1)
    p = np.array([0.3, 2.0])
    z = np.array([[[1.5, -0.5]], [[0.25, 2.0]]])
    got = orc.rope(z, p, 1e4)
    for n in range(2):
        c, s = np.cos(p[n]), np.sin(p[n])
        want = np.array([c * z[n, 0, 0] - s * z[n, 0, 1], s * z[n, 0, 0] + c * z[n, 0, 1]])
        np.testing.assert_allclose(got[n, 0], want, atol=1e-15)


def test_finite_difference_gradients():
    rng = np.random.default_rng(11)
    w = synth.make_custom_workload([[[(3, 4, 2), (2, 3, 2)]], [[(4, 0, 0)]]], hq=2, hkv=1, d=8, base=100.0)
    lay, q, k, v = _inputs(w, rng)
    do = rng.standard_normal(q.shape)
    o, lse = orc.forward(q, k, v, lay, w.base)
    dq, dk, dv = orc.backward(q, k, v, o, do, lse, lay, w.base)

    def f(qq, kk, vv):
        return float((orc.forward(qq, kk, vv, lay, w.base)[0] * do).sum())

    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[i] += eps
            xm[i] -= eps
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num[i] = (f(*args_p) - f(*args_m)) / (2 * eps)
        rel = np.linalg.norm(num - g) / np.linalg.norm(g)
        assert rel < 1e-7, (name, rel)


def test_row_and_column_samples_match_dense():
    rng = np.random.default_rng(4)
    w = synth.random_small_workload(21, hq=4, hkv=2, d=16)
    lay, q, k, v = _inputs(w, rng)
    do = rng.standard_normal(q.shape)
    o, lse = orc.attention_fwd(q, k, v, lay)
    dq, dk, dv = orc.attention_bwd(q, k, v, o, do, lse, lay)
    rows = rng.choice(lay.total, size=25, replace=False)
    got = orc.attention_rows(q, k, v, lay, rows, [0, 3], do=do)
    np.testing.assert_allclose(got["o"], o[rows][:, [0, 3]], atol=1e-12)
    np.testing.assert_allclose(got["lse"], lse[[0, 3]][:, rows], atol=1e-12)
    np.testing.assert_allclose(got["dq"], dq[rows][:, [0, 3]], atol=1e-12)
    cols = rng.choice(lay.total, size=12, replace=False)
    gk, gv = orc.attention_cols(q, k, v, do, lay, cols, kv_head=1)
    np.testing.assert_allclose(gk, dk[cols, 1], atol=1e-12)
    np.testing.assert_allclose(gv, dv[cols, 1], atol=1e-12)


def test_dv_sum_identity():
    """Rows of P sum to one, so sum_k dV[k] = sum over the group's rows of dO."""
    rng = np.random.default_rng(8)
    w = synth.random_small_workload(9, hq=4, hkv=2, d=16)
    lay, q, k, v = _inputs(w, rng)
    do = rng.standard_normal(q.shape)
    o, lse = orc.attention_fwd(q, k, v, lay)
    dq, dk, dv = orc.attention_bwd(q, k, v, o, do, lse, lay)
    for g in range(2):
        np.testing.assert_allclose(dv[:, g].sum(0), do[:, 2 * g:2 * g + 2].sum((0, 1)), atol=1e-10)
        np.testing.assert_allclose(dk[:, g].sum(0), 0.0, atol=1e-10)

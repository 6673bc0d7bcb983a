"""GPU parity of the attention forward and backward against the fp64 oracle.

Element by element at sizes the oracle evaluates densely in seconds (several
128-token tiles, ragged tails, zero-length segments, GQA, head_dim 64 and 128);
on sampled rows and keys at the full workload sizes, in the launch
configuration the benchmark times; plus properties that hold at any size.
"""

import numpy as np
import pytest
import torch

import block_sparse_masked_segment_b200 as opr
import synth
from oracle import opr_oracle as orc
from parity_helpers import assert_close, attention_order, block_map_in_order, inputs, to_dev

pytestmark = pytest.mark.gpu


def _run_gpu(w, q, k, v, do, out_dtype=torch.float32):
    att = opr.OnePassAttention(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, base=w.base)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    o, lse, qr, kr = att.forward(qd, kd, vd, out_dtype=out_dtype)
    res = dict(o=o, lse=lse)
    if do is not None:
        dq, dk, dv = att.backward(qr, kr, vd, o, to_dev(do), lse)
        res.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert opr.read_status(att.layout.dev_status) == []
    return {kk: vv.float().cpu().numpy() for kk, vv in res.items()}, att.layout


def _dense_check(w, seed, bwd=True, do_scale=1.0):
    """Element-wise parity of O, LSE (and dQ, dK, dV) with the oracle.  With do_scale the
    upstream gradient is dO * do_scale; the gradients scale with it, and so does their
    absolute tolerance (the relative one is unchanged)."""
    q, k, v, do = inputs(w, seed, with_do=bwd)
    if bwd and do_scale != 1.0:
        do = (do.astype(np.float64) * do_scale).astype(np.float32)
        do = synth.round_bf16(do)  # dO as the bf16 values the GPU receives
    got, _ = _run_gpu(w, q, k, v, do)
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    o, lse = orc.forward(q, k, v, lay, w.base)
    assert_close("O", got["o"], o)
    assert_close("LSE", got["lse"], lse)
    if bwd:
        dq, dk, dv = orc.backward(q, k, v, o, do, lse, lay, w.base)
        tol = 1e-2 * do_scale
        assert_close("dQ", got["dq"], dq, max_abs=tol)
        assert_close("dK", got["dk"], dk, max_abs=tol)
        assert_close("dV", got["dv"], dv, max_abs=tol)


@pytest.mark.parametrize("seed", range(3))
@pytest.mark.parametrize("d", [128, 64])
def test_fwd_bwd_random_ragged(seed, d):
    w = synth.random_small_workload(seed, n_seqs=2, max_convs=3, max_turns=4, hq=4, hkv=2, d=d, base=1e4)
    _dense_check(w, 100 + seed)


def test_fwd_bwd_tiny_config():
    """Tiny workload: N = 2 turns of h16 t32 r16, one head of 64, base 1e4, with fp32 Q and K as the
    workload specifies: RoPE takes them in fp32 and writes the fp16 operands of the attention
    kernels.  v and dO enter as bf16 (the kernels' operand types), so they are rounded once and the
    oracle reads the same rounded values; it reads q and k unrounded."""
    from synth import gaussian

    w = synth.make_workload(0)
    assert w.extra["fp32_inputs"]
    rng = np.random.default_rng(1000)
    n = w.total_tokens
    q, k = gaussian(rng, (n, w.hq, w.d), bf16=False), gaussian(rng, (n, w.hkv, w.d), bf16=False)
    v, do = gaussian(rng, (n, w.hkv, w.d)), gaussian(rng, (n, w.hq, w.d))
    att = opr.OnePassAttention(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, base=w.base)
    f32 = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to("cuda")  # noqa: E731
    o, lse, qr, kr = att.forward(f32(q), f32(k), to_dev(v))
    dq, dk, dv = att.backward(qr, kr, to_dev(v), o, to_dev(do), lse)
    torch.cuda.synchronize()
    assert opr.read_status(att.layout.dev_status) == []
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    ro, rlse = orc.forward(q, k, v, lay, w.base)
    rdq, rdk, rdv = orc.backward(q, k, v, ro, do, rlse, lay, w.base)
    for name, g, r in (("O", o, ro), ("LSE", lse, rlse), ("dQ", dq, rdq), ("dK", dk, rdk), ("dV", dv, rdv)):
        assert_close(name, g.cpu().numpy(), r)


@pytest.mark.parametrize("do_scale", [2.0 ** -20, 1e-6, 1e-8, 3e5])
def test_backward_at_realistic_gradient_scales(do_scale):
    """Upstream gradients far from 1 (a loss divided by the token count and passed back
    through later layers is 1e-5 .. 1e-8; 3e5 lies beyond fp16's range): the backward
    scales dO by a power of two before its fp16 copies, so the relative error stays at
    the standard and no range flag is raised."""
    w = synth.random_small_workload(23, n_seqs=2, max_convs=2, max_turns=3, hq=4, hkv=2, d=128, base=1e6)
    _dense_check(w, 230, do_scale=do_scale)


def test_fwd_bwd_gqa_8_to_1():
    w = synth.random_small_workload(7, n_seqs=1, max_convs=2, max_turns=3, hq=8, hkv=1, d=128, base=1e6)
    _dense_check(w, 7)


def test_fwd_bwd_segment_edges():
    """Segments and conversations that start and end on and next to tile edges; a 1-token sequence."""
    w = synth.make_custom_workload([
        [[(128, 128, 64)], [(127, 1, 128), (1, 127, 129)]],
        [[(1, 0, 0)]],
        [[(0, 0, 1), (3, 0, 0)], [(200, 57, 0)]],
    ], hq=2, hkv=1, d=128, base=1e4)
    _dense_check(w, 3)


def test_forward_p_v_in_fp16_and_bf16():
    """The forward's O += P V takes P in v's type.  With v in fp16 (the pipeline's choice) P keeps
    11 bits; with v in bf16, 8.  Both meet the standard on O and LSE; the fp16 form's O error is
    several times smaller (the bf16 rounding of P dominates the bf16 form's)."""
    w = synth.random_small_workload(8, n_seqs=2, max_convs=2, max_turns=4, hq=8, hkv=2, d=128, base=1e4)
    q, k, v, _ = inputs(w, 4200, with_do=False)
    lo = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    o_ref, lse_ref = orc.forward(q, k, v, lo, w.base)
    att = opr.OnePassAttention(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, base=w.base)
    o16, lse16, qr, kr = att.forward(to_dev(q), to_dev(k), to_dev(v))  # fp16 copy of v inside
    v_bf = torch.empty((w.total_tokens, w.hkv, w.d), dtype=torch.bfloat16, device="cuda")
    opr.opr_rope(to_dev(v), None, w.base, out=v_bf, row_map=att.layout.attn_pos)  # bf16 v, attention order
    o_bf, lse_bf = opr.opr_attn_fwd(qr, kr, v_bf, att.layout)
    torch.cuda.synchronize()
    assert opr.read_status(att.layout.dev_status) == []
    e16, _ = assert_close("O (fp16 P)", o16.cpu().numpy(), o_ref)
    ebf, _ = assert_close("O (bf16 P)", o_bf.cpu().numpy(), o_ref)
    assert_close("LSE (fp16 P)", lse16.cpu().numpy(), lse_ref)
    assert_close("LSE (bf16 P)", lse_bf.cpu().numpy(), lse_ref)
    np.testing.assert_array_equal(lse16.cpu().numpy(), lse_bf.cpu().numpy())  # P's type does not enter LSE
    assert e16 < ebf / 3, (e16, ebf)


def test_fwd_bf16_output_is_rounded_fp32():
    w = synth.random_small_workload(11, hq=2, hkv=1, d=128)
    q, k, v, _ = inputs(w, 11, with_do=False)
    g32, _ = _run_gpu(w, q, k, v, None, torch.float32)
    g16, _ = _run_gpu(w, q, k, v, None, torch.bfloat16)
    np.testing.assert_array_equal(g16["o"], synth.round_bf16(g32["o"]))


def test_theorem_2_1_on_gpu_path():
    """The N-pass runs of the same conversations through the same kernels give the
    one-pass rows of t_i and r_i^out (and of h_j, r_j^in) within the float standard."""
    w = synth.random_small_workload(5, n_seqs=1, max_convs=2, max_turns=4, hq=4, hkv=2, d=128, base=1e6)
    q, k, v, _ = inputs(w, 5, with_do=False)
    one, _ = _run_gpu(w, q, k, v, None)
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    lists = orc.npass_token_lists(lay, w.turn_lens, w.conv_turn_ptr)
    idx = np.concatenate([t for _, _, t in lists])
    nw, origin = synth.npass_workload(w)
    assert [(c, i) for c, i, _ in lists] == origin
    many, _ = _run_gpu(nw, q[idx], k[idx], v[idx], None)
    assert_close("O one-pass vs N-pass", one["o"][idx], many["o"])
    assert_close("LSE one-pass vs N-pass", one["lse"][:, idx], many["lse"])


# ---------------------------------------------------------------- full sizes

def _sample_rows(lay, rng, n):
    return np.sort(rng.choice(lay.total, size=min(n, lay.total), replace=False))


def _tail_keys(lay, rng, n, tail=24):
    """Keys among the last `tail` tokens of the r^in and r^out segments of each
    conversation's last turn: only a few rows see them, so the oracle can
    evaluate their column sums exactly."""
    keys = []
    for c in np.unique(lay.conv_idx):
        sel = np.nonzero(lay.conv_idx == c)[0]
        last = sel[lay.turn_idx[sel] == lay.turn_idx[sel].max()]
        for typ in (orc.RIN, orc.ROUT):
            seg = last[lay.token_type[last] == typ]
            keys.append(seg[-tail:])
    keys = np.concatenate(keys)
    return np.sort(rng.choice(keys, size=min(n, len(keys)), replace=False))


def _dk_sum_post_rope(dk_pre, lay, base, kv_head):
    """Rows of dS sum to zero, so the keys' gradients w.r.t. the rotated k sum to zero."""
    post = orc.rope(dk_pre[:, kv_head:kv_head + 1, :].astype(np.float64), lay.pos_id, base)[:, 0]
    return np.abs(post.sum(0)).max() / np.abs(post).sum(0).max()


@pytest.mark.parametrize("config", [1, 2, 4])
def test_full_size_sampled(config):
    w = synth.make_workload(config)
    bwd = config != 1
    q, k, v, do = inputs(w, 1000 + config, with_do=bwd)
    got, _ = _run_gpu(w, q, k, v, do, out_dtype=torch.bfloat16)  # O stored as the benchmark stores it
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    qr = orc.rope(q, lay.pos_id, w.base)
    kr = orc.rope(k, lay.pos_id, w.base)
    rng = np.random.default_rng(config)
    rows = _sample_rows(lay, rng, 256)
    heads = sorted(rng.choice(w.hq, size=4, replace=False).tolist())
    ref = orc.attention_rows(qr, kr, v, lay, rows, heads, do=do if bwd else None)
    assert_close("O rows", got["o"][rows][:, heads], ref["o"])
    assert_close("LSE rows", got["lse"][heads][:, rows], ref["lse"])
    if not bwd:
        return
    # dQ of sampled rows (w.r.t. the unrotated q): rotate the oracle's back
    dq_rows = orc.rope(ref["dq"], lay.pos_id[rows], w.base, inverse=True)
    assert_close("dQ rows", got["dq"][rows][:, heads], dq_rows)
    keys = _tail_keys(lay, rng, 48)
    if config == 2:
        keys = np.union1d(keys, _first_turn_keys(lay, w, rng, 24))
    g = int(rng.integers(w.hkv))
    dk, dv = orc.attention_cols(qr, kr, v, do, lay, keys, kv_head=g)
    dk = orc.rope(dk[:, None, :], lay.pos_id[keys], w.base, inverse=True)[:, 0]
    assert_close("dK keys", got["dk"][keys, g], dk)
    assert_close("dV keys", got["dv"][keys, g], dv)
    # rows of P sum to one: sum over keys of dV equals the sum of dO over the group's rows
    grp = w.hq // w.hkv
    for gg in range(w.hkv):
        want = do[:, gg * grp:(gg + 1) * grp].astype(np.float64).sum((0, 1))
        np.testing.assert_allclose(got["dv"][:, gg].astype(np.float64).sum(0), want, atol=0.5, rtol=2e-3)
    assert _dk_sum_post_rope(got["dk"], lay, w.base, g) < 1e-3


@pytest.mark.parametrize("n_turns", [2, 8, 16])
def test_depth_sweep_sampled(n_turns):
    w = synth.make_workload(3, n_turns=n_turns)
    q, k, v, do = inputs(w, 3000 + n_turns)
    got, _ = _run_gpu(w, q, k, v, do, out_dtype=torch.bfloat16)
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    qr = orc.rope(q, lay.pos_id, w.base)
    kr = orc.rope(k, lay.pos_id, w.base)
    rng = np.random.default_rng(n_turns)
    rows = _sample_rows(lay, rng, 192)
    heads = [0, 13, 31]
    ref = orc.attention_rows(qr, kr, v, lay, rows, heads, do=do)
    assert_close("O rows", got["o"][rows][:, heads], ref["o"])
    assert_close("LSE rows", got["lse"][heads][:, rows], ref["lse"])
    assert_close("dQ rows", got["dq"][rows][:, heads], orc.rope(ref["dq"], lay.pos_id[rows], w.base, inverse=True))
    keys = _tail_keys(lay, rng, 32)
    dk, dv = orc.attention_cols(qr, kr, v, do, lay, keys, kv_head=5)
    dk = orc.rope(dk[:, None, :], lay.pos_id[keys], w.base, inverse=True)[:, 0]
    assert_close("dK keys", got["dk"][keys, 5], dk)
    assert_close("dV keys", got["dv"][keys, 5], dv)


def test_full_kv_group_depth_sweep_4_turns():
    """Every dQ, dK and dV element of one GQA group (4 q heads, 1 kv head) on the depth-sweep
    conversation of 4 turns (4,608 tokens), against the dense oracle backward of that group:
    every key's gradient sums over all the query tiles and q heads that see it."""
    w = synth.make_workload(3, n_turns=4)
    q, k, v, do = inputs(w, 3004)
    got, _ = _run_gpu(w, q, k, v, do)
    grp = w.hq // w.hkv
    g = 3
    hs = slice(g * grp, (g + 1) * grp)
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    qg, kg, vg, dog = q[:, hs], k[:, g:g + 1], v[:, g:g + 1], do[:, hs]
    o, lse = orc.forward(qg, kg, vg, lay, w.base)
    dq, dk, dv = orc.backward(qg, kg, vg, o, dog, lse, lay, w.base)
    assert_close("O group", got["o"][:, hs], o)
    assert_close("dQ group", got["dq"][:, hs], dq)
    assert_close("dK group", got["dk"][:, g:g + 1], dk)
    assert_close("dV group", got["dv"][:, g:g + 1], dv)


def _first_turn_keys(lay, w, rng, n):
    """h and r^in keys of the first turn of the shortest conversation with at least three
    turns: every later row of the conversation sees them, so their gradients are the longest
    sums of the layer."""
    conv_turns = np.diff(w.conv_turn_ptr)
    conv_len = [int((lay.conv_idx == c).sum()) for c in range(w.n_convs)]
    c = min((c for c in range(w.n_convs) if conv_turns[c] >= 3), key=lambda c: conv_len[c])
    sel = np.nonzero((lay.conv_idx == c) & (lay.turn_idx == 0))[0]
    keys = sel[(lay.token_type[sel] == orc.H) | (lay.token_type[sel] == orc.RIN)]
    return np.sort(rng.choice(keys, size=min(n, len(keys)), replace=False))


@pytest.mark.parametrize("d", [128, 64])
def test_backward_with_positions_equals_rotation_afterwards(d):
    """opr_attn_bwd given the position ids returns dq and dk w.r.t. the unrotated q and k:
    exactly the rotated-frame gradients followed by opr_rope(inverse)."""
    w = synth.random_small_workload(17, n_seqs=2, max_convs=3, max_turns=4, hq=4, hkv=2, d=d, base=1e6)
    q, k, v, do = inputs(w, 17)
    att = opr.OnePassAttention(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, base=w.base)
    qd, kd, vd, dod = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    o, lse, qr, kr = att.forward(qd, kd, vd)
    lay = att.layout
    dq0, dk0, dv0 = opr.opr_attn_bwd(qr, kr, vd, o, dod, lse, lay)
    opr.opr_rope(dq0, lay.pos_id, w.base, inverse=True)
    opr.opr_rope(dk0, lay.pos_id, w.base, inverse=True)
    dq1, dk1, dv1 = opr.opr_attn_bwd(qr, kr, vd, o, dod, lse, lay, rope_base=w.base)
    torch.cuda.synchronize()
    assert opr.read_status(lay.dev_status) == []
    for name, a, b in (("dQ", dq0, dq1), ("dK", dk0, dk1), ("dV", dv0, dv1)):
        np.testing.assert_array_equal(b.cpu().numpy(), a.cpu().numpy(), err_msg=name)


@pytest.mark.parametrize("case", ["ragged_8q2kv", "gqa_8q1kv", "depth4_32q8kv"])
def test_dkdv_split_by_q_head_and_unsplit_agree(case):
    """Short dK/dV grids (few key tiles x kv heads) split their long key columns by q head:
    per-head partials in the workspace, then a group sum.  A workspace of the minimum size keeps
    the stage unsplit.  Both
    forms match the oracle; they differ from each other only by the order of the fp32 group sum
    (a few 1e-6 of the largest gradient, far inside the oracle tolerance; dQ, which the split
    does not touch, is bit-identical)."""
    if case == "ragged_8q2kv":
        w = synth.random_small_workload(5, n_seqs=2, max_convs=2, max_turns=4, hq=8, hkv=2, d=128, base=1e4)
    elif case == "gqa_8q1kv":
        w = synth.random_small_workload(6, n_seqs=1, max_convs=2, max_turns=3, hq=8, hkv=1, d=128, base=1e4)
    else:
        w = synth.make_workload(3, n_turns=4)
    q, k, v, do = inputs(w, 4100)
    att = opr.OnePassAttention(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, base=w.base)
    qd, kd, vd, dod = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    o, lse, qr, kr = att.forward(qd, kd, vd)
    lay = att.layout
    assert w.hq > w.hkv and lay.n_seqs * lay.T * w.hkv < 4 * 148  # a grid the split applies to
    full = opr.opr_attn_bwd_workspace_bytes(lay.n_seqs, lay.max_seqlen, w.hq, w.d)
    least = opr.opr_attn_bwd_min_workspace_bytes(lay.n_seqs, lay.max_seqlen, w.hq, w.d)
    assert full > least
    ws_full = torch.full((full,), 0xFF, dtype=torch.uint8, device="cuda")
    split = opr.opr_attn_bwd(qr, kr, vd, o, dod, lse, lay, workspace=ws_full, rope_base=w.base)
    unsplit = opr.opr_attn_bwd(qr, kr, vd, o, dod, lse, lay, rope_base=w.base,
                               workspace=torch.empty(least, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    assert opr.read_status(lay.dev_status) == []
    # the split form ran on the long columns (seen by >= 2T / group query tiles, include/opr.h):
    # it wrote per-head partials past the minimum workspace
    lo = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    col_cnt = ((block_map_in_order(lo, attention_order(lo)) & 3) > 0).sum(axis=1)  # [n_seqs, key tile]
    min_cnt = -(-2 * lay.T // (w.hq // w.hkv))
    assert int(col_cnt.max()) >= min_cnt
    assert bool((ws_full[least:] != 0xFF).any())
    split = [t.cpu().numpy() for t in split]
    unsplit = [t.cpu().numpy() for t in unsplit]
    np.testing.assert_array_equal(split[0], unsplit[0], err_msg="dQ")
    for name, a, b in zip(("dK", "dV"), split[1:], unsplit[1:]):
        np.testing.assert_allclose(a, b, rtol=1e-4, atol=2e-5 * float(np.abs(b).max()), err_msg=name)
    if case == "depth4_32q8kv":  # one GQA group densely (the whole problem is too large for the oracle)
        grp = w.hq // w.hkv
        g = 5
        hs = slice(g * grp, (g + 1) * grp)
        qg, kg, vg, dog = q[:, hs], k[:, g:g + 1], v[:, g:g + 1], do[:, hs]
        oo, ll = orc.forward(qg, kg, vg, lo, w.base)
        ref = orc.backward(qg, kg, vg, oo, dog, ll, lo, w.base)
        got = [split[0][:, hs], split[1][:, g:g + 1], split[2][:, g:g + 1]]
    else:
        oo, ll = orc.forward(q, k, v, lo, w.base)
        ref = orc.backward(q, k, v, oo, do, ll, lo, w.base)
        got = split
    for name, g_, r in zip(("dQ", "dK", "dV"), got, ref):
        assert_close(name, g_, r)


def test_deterministic_backward():
    w = synth.random_small_workload(2, hq=4, hkv=2, d=128)
    q, k, v, do = inputs(w, 2)
    a, _ = _run_gpu(w, q, k, v, do)
    b, _ = _run_gpu(w, q, k, v, do)
    for name in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_array_equal(a[name], b[name])


@pytest.mark.parametrize("where", ["v", "do"])
def test_backward_flags_values_fp16_cannot_hold(where):
    """The dK/dV products read fp16 copies of v and of the scaled dO: a |v| beyond 65504,
    or a non-finite dO, is reported in the status word, never silently clipped."""
    from block_sparse_masked_segment_b200 import _abi

    w = synth.random_small_workload(4, hq=4, hkv=2, d=128)
    q, k, v, do = inputs(w, 4)
    if where == "v":
        v = v.copy()
        v[w.total_tokens // 2, 1, 7] = 1.0e5
    else:
        do = do.copy()
        do[w.total_tokens // 2, 1, 7] = np.inf
    att = opr.OnePassAttention(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, base=w.base)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    o, lse, qr, kr = att.forward(qd, kd, vd)
    att.backward(qr, kr, vd, o, to_dev(do), lse)
    torch.cuda.synchronize()
    assert opr.read_status(att.layout.dev_status) == [_abi.DEV_BITS[16]]


def test_backward_in_range_values_leave_status_clear():
    """A large finite dO (|dO| = 6e4 everywhere, scaled down before its fp16 copy) raises no flag."""
    w = synth.random_small_workload(5, hq=4, hkv=2, d=64)
    q, k, v, do = inputs(w, 5)
    do = do * 0 + np.float32(6.0e4) * np.sign(do)
    att = opr.OnePassAttention(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, base=w.base)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    o, lse, qr, kr = att.forward(qd, kd, vd)
    att.backward(qr, kr, vd, o, to_dev(do), lse)
    torch.cuda.synchronize()
    assert opr.read_status(att.layout.dev_status) == []

"""GPU parity of the K-pass arrangement (opr_kpass: plan and token map) against
the oracle, and Theorem 2.1 through it on the GPU attention path."""

import numpy as np
import pytest
import torch

import block_sparse_masked_segment_b200 as opr
import synth
from oracle import opr_oracle as orc
from parity_helpers import assert_close, to_dev

pytestmark = pytest.mark.gpu


def _check(w, K):
    kp = opr.opr_kpass(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, K)
    torch.cuda.synchronize()
    assert opr.read_status(kp.dev_status) == []
    l2, c2, s2, tsrc = orc.kpass_plan(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, K)
    np.testing.assert_array_equal(kp.turn_lens.cpu().numpy(), l2)
    np.testing.assert_array_equal(kp.conv_turn_ptr.cpu().numpy(), c2)
    np.testing.assert_array_equal(kp.seq_conv_ptr.cpu().numpy(), s2)
    np.testing.assert_array_equal(kp.turn_src.cpu().numpy(), tsrc)
    src, copies = orc.kpass_index(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, K)
    np.testing.assert_array_equal(kp.src_index.cpu().numpy(), src)
    np.testing.assert_array_equal(kp.copy_index.cpu().numpy(), copies)
    return kp, (l2, c2, s2), src, copies


@pytest.mark.parametrize("K", [1, 2, 3, 4])
@pytest.mark.parametrize("seed", [0, 1])
def test_plan_and_map_random(K, seed):
    _check(synth.random_small_workload(seed, n_seqs=2, max_convs=3, max_turns=6), K)


def test_plan_and_map_full_size_k2():
    _check(synth.make_workload(2), 2)


def test_fold_over_k_plus_one_slots():
    w = synth.random_small_workload(4, max_turns=6)
    kp, _, src, copies = _check(w, 3)
    dy = np.random.default_rng(0).standard_normal((len(src), 40)).astype(np.float32)
    got = opr.opr_fold_rows(torch.from_numpy(dy).cuda(), kp.copy_index).cpu().numpy()
    np.testing.assert_array_equal(got, orc.fold_rows(dy, copies))


@pytest.mark.parametrize("K", [2, 3])
def test_theorem_2_1_through_k_pass_on_gpu(K):
    """Attention over the K-pass arrangement (inputs gathered by the map): every copy's O row
    matches the oracle's one-pass row of that token (context copies the h / r^in row)."""
    w = synth.random_small_workload(6, n_seqs=1, max_convs=2, max_turns=5, hq=4, hkv=2, d=64)
    kp, (l2, c2, s2), src, copies = _check(w, K)
    rng = np.random.default_rng(1)
    n_orig = copies.shape[0]
    q0 = synth.round_bf16(rng.standard_normal((n_orig, w.hq, w.d)).astype(np.float32))
    k0 = synth.round_bf16(rng.standard_normal((n_orig, w.hkv, w.d)).astype(np.float32))
    v0 = synth.round_bf16(rng.standard_normal((n_orig, w.hkv, w.d)).astype(np.float32))
    att = opr.OnePassAttention(l2, c2, s2, base=w.base)
    gq, gk, gv = (opr.opr_gather_rows(to_dev(x), kp.src_index) for x in (q0, k0, v0))
    o_k, _, _, _ = att.forward(gq, gk, gv, out_dtype=torch.float32)
    torch.cuda.synchronize()
    d_src, d_copies = orc.duplication_index(w.turn_lens, w.conv_turn_ptr)
    lay1 = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    o1, _ = orc.forward(q0[d_src], k0[d_src], v0[d_src], lay1, w.base)
    got, ref = [], []
    ok = o_k.cpu().numpy()
    for o in range(n_orig):
        for slot, p in enumerate(copies[o]):
            if p >= 0:
                got.append(ok[p])
                ref.append(o1[d_copies[o, 1] if slot == 1 else d_copies[o, 0]])
    assert_close("O rows of K-pass copies", np.stack(got), np.stack(ref))

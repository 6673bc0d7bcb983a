"""GPU parity of the loss side (opr_loss_rows, opr_cross_entropy) against the oracle."""

import numpy as np
import pytest
import torch

import block_sparse_masked_segment_b200 as opr
from block_sparse_masked_segment_b200 import _abi
import synth
from oracle import opr_oracle as orc

pytestmark = pytest.mark.gpu


def _check_rows(w):
    rows, targets = opr.opr_loss_rows(w.turn_lens)
    torch.cuda.synchronize()
    assert opr.read_status(rows._inputs[1]) == []
    r_rows, r_targets = orc.loss_rows(w.turn_lens, w.conv_turn_ptr)
    np.testing.assert_array_equal(rows.cpu().numpy(), r_rows)
    np.testing.assert_array_equal(targets.cpu().numpy(), r_targets)
    return rows, targets


def test_worked_example_rows():
    rows, targets = _check_rows(synth.make_custom_workload([[[[2, 3, 2], [1, 2, 1]]]]))
    assert rows.cpu().tolist() == [1, 2, 3, 4, 7, 9, 10, 11]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_rows_random_ragged(seed):
    _check_rows(synth.random_small_workload(seed, n_seqs=3, max_convs=4, max_turns=5))


def test_rows_many_turns_and_full_size():
    rng = np.random.default_rng(5)
    convs = [[[int(a), int(b), int(c)] for a, b, c in rng.integers(0, 6, size=(n, 3))] for n in rng.integers(1, 30, 80)]
    _check_rows(synth.make_custom_workload([convs]))
    _check_rows(synth.make_workload(2))


@pytest.mark.parametrize("V", [5003, 5008])  # scalar path, 16-byte path
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_cross_entropy_matches_oracle(dtype, V):
    rng = np.random.default_rng(0)
    n = 37
    z = (rng.standard_normal((n, V)) * 4).astype(np.float32)
    tgt = rng.integers(0, V, size=n).astype(np.int32)
    tgt[3] = -1  # ignored row
    zd = torch.from_numpy(z).to("cuda", dtype)
    zr = zd.float().cpu().numpy().astype(np.float64)  # the values the kernel reads
    loss, dl = opr.opr_cross_entropy(zd, torch.from_numpy(tgt).cuda(), grad_scale=0.5)
    torch.cuda.synchronize()
    assert opr.read_status(loss._status) == []
    keep = tgt >= 0
    r_loss, r_dz = orc.cross_entropy(zr[keep], tgt[keep])
    got = loss.cpu().numpy()
    np.testing.assert_allclose(got[keep], r_loss, rtol=2e-6, atol=2e-5)
    assert got[3] == 0.0
    g = dl.float().cpu().numpy()
    assert not g[3].any()
    tol = 1e-6 if dtype == torch.float32 else 0.5 * 2.0 ** -8  # bf16 output: one rounding
    np.testing.assert_allclose(g[keep], 0.5 * r_dz, atol=tol, rtol=tol)


def test_cross_entropy_with_masked_logits():
    """-inf logits (a masked vocabulary entry) contribute nothing and get a zero gradient."""
    z = torch.randn(4, 64, device="cuda")
    z[:, 5] = float("-inf")
    tgt = torch.tensor([0, 1, 2, 3], dtype=torch.int32, device="cuda")
    loss, dl = opr.opr_cross_entropy(z, tgt)
    zz = z.clone()
    zz[:, 5] = -1e30
    ref = torch.nn.functional.cross_entropy(zz.double(), tgt.long(), reduction="none")
    torch.testing.assert_close(loss.double(), ref, rtol=1e-5, atol=1e-5)
    assert bool((dl[:, 5] == 0).all())


def test_cross_entropy_flags_target_beyond_vocab():
    z = torch.zeros((2, 10), device="cuda")
    loss, _ = opr.opr_cross_entropy(z, torch.tensor([3, 10], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert opr.read_status(loss._status) == [_abi.DEV_BITS[1]]
    assert loss.cpu().tolist() == [pytest.approx(np.log(10.0)), 0.0]


def test_toy_model_loss_through_the_gpu_loss_side():
    """The oracle toy transformer's one-pass logits, pushed through opr_loss_rows and
    opr_cross_entropy on the GPU, give the N-pass losses (fp32 tolerance)."""
    from test_oracle_loss import ToyModel

    w = synth.random_small_workload(1, n_seqs=1, max_convs=2, max_turns=4, h=(0, 9), t=(0, 9), r=(0, 9))
    model = ToyModel(seed=1)
    lens = np.asarray(w.turn_lens).reshape(-1, 3)
    ids = np.random.default_rng(11).integers(0, model.V, size=int(lens.sum()))
    src, _ = orc.duplication_index(w.turn_lens, w.conv_turn_ptr)
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    z = model.logits(ids[src], lambda q, k, v: orc.forward(q, k, v, lay, 1e4)[0])
    rows, targets = _check_rows(w)
    zr = torch.from_numpy(z.astype(np.float32)).cuda()[rows.long()].contiguous()
    tid = torch.from_numpy(ids.astype(np.int32)).cuda()[targets.long()].contiguous()
    loss, _ = opr.opr_cross_entropy(zr, tid, with_grad=False)
    r_rows, r_targets = orc.loss_rows(w.turn_lens, w.conv_turn_ptr)
    ref, _ = orc.cross_entropy(z[r_rows], ids[r_targets])
    np.testing.assert_allclose(loss.cpu().numpy(), ref, rtol=1e-5, atol=1e-5)

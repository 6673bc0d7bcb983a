"""GPU parity of the token-duplication step (opr_duplication_index, opr_gather_rows,
opr_fold_rows) against the oracle: index maps bit-exact, row copies exact, the
fp32 fold bit-exact (first copy + second copy, the oracle's order)."""

import numpy as np
import pytest
import torch

import block_sparse_masked_segment_b200 as opr
from block_sparse_masked_segment_b200 import _abi
import synth
from oracle import opr_oracle as orc

pytestmark = pytest.mark.gpu


def _check_maps(w):
    src, copies = opr.opr_duplication_index(w.turn_lens, w.conv_turn_ptr)
    status = src._inputs[2]
    torch.cuda.synchronize()
    assert opr.read_status(status) == []
    r_src, r_copies = orc.duplication_index(w.turn_lens, w.conv_turn_ptr)
    np.testing.assert_array_equal(src.cpu().numpy(), r_src)
    np.testing.assert_array_equal(copies.cpu().numpy(), r_copies)
    return src, copies, r_src, r_copies


def test_worked_example():
    w = synth.make_custom_workload([[[[2, 3, 2], [1, 2, 1]]]])
    src, copies, _, _ = _check_maps(w)
    assert src.cpu().tolist() == [0, 1, 2, 3, 4, 5, 6, 5, 6, 7, 8, 9, 10, 10]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_maps_random_ragged(seed):
    _check_maps(synth.random_small_workload(seed, n_seqs=3, max_convs=4, max_turns=5))


def test_maps_zero_length_segments():
    _check_maps(synth.make_custom_workload([[[[0, 3, 2], [2, 0, 0], [1, 1, 0], [0, 0, 3]]], [[[4, 0, 1]]]]))


def test_maps_many_turns_across_chunks():
    """More turns than one scan chunk (1024) of the single-block kernel."""
    rng = np.random.default_rng(7)
    convs = [[[int(a), int(b), int(c)] for a, b, c in rng.integers(0, 9, size=(n, 3))] for n in rng.integers(1, 40, 90)]
    _check_maps(synth.make_custom_workload([convs]))


@pytest.mark.parametrize("config", [1, 2])
def test_maps_full_size(config):
    _check_maps(synth.make_workload(config))


def test_gather_and_fold_rows():
    w = synth.random_small_workload(11, n_seqs=2)
    src, copies, r_src, r_copies = _check_maps(w)
    n_orig = r_copies.shape[0]
    rng = np.random.default_rng(3)
    # token ids (4-byte rows), bf16 hidden rows (16-byte path), 3-byte rows (byte path)
    ids = rng.integers(0, 150000, size=(n_orig,)).astype(np.int32)
    got = opr.opr_gather_rows(torch.from_numpy(ids).cuda(), src).cpu().numpy()
    np.testing.assert_array_equal(got, ids[r_src])
    hid = synth.round_bf16(rng.standard_normal((n_orig, 256)).astype(np.float32))
    hid_d = torch.from_numpy(hid).to("cuda", torch.bfloat16)
    got = opr.opr_gather_rows(hid_d, src).float().cpu().numpy()
    np.testing.assert_array_equal(got, orc.gather_rows(hid, r_src))
    small = rng.integers(0, 255, size=(n_orig, 3)).astype(np.uint8)
    got = opr.opr_gather_rows(torch.from_numpy(small).cuda(), src).cpu().numpy()
    np.testing.assert_array_equal(got, small[r_src])
    # fp32 fold, float4 path (width 256) and scalar path (width 3)
    for width in (256, 3):
        dy = rng.standard_normal((len(r_src), width)).astype(np.float32)
        got = opr.opr_fold_rows(torch.from_numpy(dy).cuda(), copies).cpu().numpy()
        np.testing.assert_array_equal(got, orc.fold_rows(dy, r_copies))


def test_fold_of_gather_counts_copies():
    w = synth.random_small_workload(12)
    src, copies, _, r_copies = _check_maps(w)
    x = torch.randn(r_copies.shape[0], 64, device="cuda")
    got = opr.opr_fold_rows(opr.opr_gather_rows(x, src), copies)
    mult = torch.from_numpy(np.where(r_copies[:, 1] >= 0, 2.0, 1.0).astype(np.float32)).cuda()[:, None]
    torch.testing.assert_close(got, x * mult, rtol=0, atol=0)


def test_total_mismatch_is_flagged_without_overrun():
    """A total smaller than the lengths give: flagged, and nothing is written past the buffers."""
    w = synth.random_small_workload(13)
    total = w.total_tokens
    orig = int(np.asarray(w.turn_lens).reshape(-1, 3).sum())
    guard = 64
    buf_src = torch.full((total - 5 + guard,), -7, dtype=torch.int32, device="cuda")
    buf_cp = torch.full(((orig - 5) * 2 + guard,), -7, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tl = torch.as_tensor(np.asarray(w.turn_lens, dtype=np.int32).reshape(-1)).cuda()
    cp = torch.as_tensor(np.asarray(w.conv_turn_ptr, dtype=np.int32)).cuda()
    lib = opr.load_library()
    st = lib.opr_duplication_index(tl.data_ptr(), cp.data_ptr(), cp.numel() - 1, tl.numel() // 3, total - 5, orig - 5,
                                   buf_src.data_ptr(), buf_cp.data_ptr(), status.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    assert _abi.DEV_BITS[2] in opr.read_status(status)
    assert bool((buf_src[total - 5:] == -7).all()) and bool((buf_cp[(orig - 5) * 2:] == -7).all())


def test_binding_rejects_bad_index_and_out_tensors():
    """The binding refuses, before any launch, index tensors of the wrong type or rank and
    output buffers of the wrong type or shape (the library would read or write past them)."""
    w = synth.random_small_workload(14)
    src, copies, _, r_copies = _check_maps(w)
    n_orig = r_copies.shape[0]
    x = torch.randn(n_orig, 8, device="cuda")
    dy = torch.randn(src.numel(), 8, device="cuda")
    with pytest.raises(opr.OprError):
        opr.opr_gather_rows(x, src.long())
    with pytest.raises(opr.OprError):
        opr.opr_fold_rows(dy, copies.long())
    with pytest.raises(opr.OprError):
        opr.opr_fold_rows(dy, copies.reshape(-1))
    with pytest.raises(opr.OprError):
        opr.opr_fold_rows(dy, copies, out=torch.empty(n_orig - 1, 8, device="cuda"))
    with pytest.raises(opr.OprError):
        opr.opr_fold_rows(dy, copies, out=torch.empty(n_orig, 8, device="cuda", dtype=torch.float16))
    torch.testing.assert_close(opr.opr_fold_rows(dy, copies, out=torch.empty(n_orig, 8, device="cuda")),
                               opr.opr_fold_rows(dy, copies), rtol=0, atol=0)

"""GPU parity of opr_build_layout and opr_rope against the oracle.

Layout, position ids, the block map and its key-half bits must match bit for
bit (One-Pass to Reason, "Token 复制", "位置 ID 策略", "分块稀疏注意力掩码").
So must the attention order (each token's row for the attention calls) and the
internal tile lists the attention kernels walk, which describe the oracle's mask
with rows and columns taken in that order.
"""

import numpy as np
import pytest
import torch

import block_sparse_masked_segment_b200 as opr
from block_sparse_masked_segment_b200 import _abi
import synth
from oracle import opr_oracle as orc
from parity_helpers import attention_order, block_map_in_order

pytestmark = pytest.mark.gpu


def _internal_block_map(lay):
    """The attention kernels' block map, read back from the layout's row lists
    (entries (J << 4) | block-map byte of the non-empty tiles of each tile row)."""
    off = opr.layout_table_offsets(lay)
    T, n_tiles = lay.T, lay.n_seqs * lay.T
    ws = lay.workspace.cpu().numpy()
    cnt = ws[off["row_cnt"]:off["row_cnt"] + 4 * n_tiles].view(np.int32)
    lists = ws[off["row_list"]:off["row_list"] + 4 * n_tiles * T].view(np.int32).reshape(n_tiles, T)
    bm = np.zeros((lay.n_seqs, T, T), dtype=np.uint8)
    for row in range(n_tiles):
        s, i = divmod(row, T)
        for e in lists[row, :cnt[row]]:
            bm[s, i, e >> 4] = e & 15
    return bm


def _compare_layout(w, internal=True):
    lay = opr.opr_build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    ref = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    torch.cuda.synchronize()
    assert opr.read_status(lay.dev_status) == []
    np.testing.assert_array_equal(lay.cu_seqlens.cpu().numpy(), ref.cu_seqlens)
    np.testing.assert_array_equal(lay.token_type.cpu().numpy(), ref.token_type)
    np.testing.assert_array_equal(lay.turn_idx.cpu().numpy(), ref.turn_idx)
    np.testing.assert_array_equal(lay.conv_idx.cpu().numpy(), ref.conv_idx)
    np.testing.assert_array_equal(lay.pos_id.cpu().numpy(), ref.pos_id)
    bm = lay.block_map.cpu().numpy()
    # each byte: tile class in bits 0-1, key halves that some query sees in bits 2-3
    np.testing.assert_array_equal(bm & 3, orc.block_map(ref, max_seqlen=lay.max_seqlen))
    np.testing.assert_array_equal(bm >> 2, orc.key_half_map(ref, max_seqlen=lay.max_seqlen))
    # attention order: attn_pos is the inverse of the order (stream index of each position)
    order = attention_order(ref)
    expect_pos = np.empty_like(order)
    expect_pos[order] = np.arange(len(order))
    np.testing.assert_array_equal(lay.attn_pos.cpu().numpy(), expect_pos)
    if internal:
        np.testing.assert_array_equal(_internal_block_map(lay), block_map_in_order(ref, order))
    return lay, ref


@pytest.mark.parametrize("seed", range(6))
def test_layout_random_ragged(seed):
    w = synth.random_small_workload(seed, n_seqs=3, max_convs=4, max_turns=5)
    _compare_layout(w)


def test_layout_zero_lengths_and_tiny_segments():
    w = synth.make_custom_workload([
        [[(0, 0, 1), (1, 0, 0), (0, 3, 0)], [(2, 2, 2)]],
        [[(5, 0, 0)]],
        [[(130, 0, 0)], [(1, 1, 1), (0, 0, 0), (127, 129, 1)]],
    ])
    _compare_layout(w)


def test_layout_block_boundaries():
    """Segments ending exactly on and just off the 128-token tile edges."""
    w = synth.make_custom_workload([
        [[(128, 128, 64)], [(127, 1, 128), (1, 127, 129)]],
        [[(256, 0, 0)], [(128, 0, 0)]],
    ])
    _compare_layout(w)


@pytest.mark.parametrize("config", [0, 1, 2, 4])
def test_layout_full_configs(config):
    w = synth.make_workload(config)
    _compare_layout(w)


@pytest.mark.parametrize("n_turns", synth.DEPTH_SWEEP_TURNS)
def test_layout_depth_sweep(n_turns):
    _compare_layout(synth.make_workload(3, n_turns=n_turns))


def test_layout_npass_is_causal():
    w, _ = synth.npass_workload(synth.make_workload(1))
    lay, ref = _compare_layout(w)
    bm = lay.block_map.cpu().numpy() & 3
    for s in range(lay.n_seqs):
        L = int(ref.cu_seqlens[s + 1] - ref.cu_seqlens[s])
        nt = (L + 127) // 128
        for I in range(nt):
            # causal: strictly below the diagonal is full, except in a tail tile row
            # (rows past the end count as not visible), which is partial
            below = 1 if (I + 1) * 128 <= L else 2
            assert all(bm[s, I, J] == below for J in range(I))
            assert bm[s, I, I] == 2
            assert all(bm[s, I, J] == 0 for J in range(I + 1, bm.shape[1]))


def test_layout_device_status_total_mismatch():
    w = synth.random_small_workload(3)
    lay = opr.opr_build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr,
                               total_tokens=w.total_tokens + 5, max_seqlen=w.max_seqlen)
    torch.cuda.synchronize()
    assert "total mismatch" in opr.read_status(lay.dev_status)


def test_layout_device_status_seq_too_long():
    w = synth.random_small_workload(4)
    lay = opr.opr_build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr,
                               total_tokens=w.total_tokens, max_seqlen=max(w.max_seqlen - 1, 1))
    torch.cuda.synchronize()
    assert "sequence longer than max_seqlen" in opr.read_status(lay.dev_status)


@pytest.mark.parametrize("in_dtype,out_dtype", [(torch.float32, torch.float32), (torch.bfloat16, torch.bfloat16),
                                                (torch.bfloat16, torch.float16), (torch.float16, torch.float16)])
@pytest.mark.parametrize("d", [64, 128])
def test_rope_parity(in_dtype, out_dtype, d):
    w = synth.make_workload(4)  # positions up to ~1.4e4
    ref_lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    lay = opr.opr_build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    rng = np.random.default_rng(0)
    x = rng.standard_normal((lay.total, 2, d)).astype(np.float32)
    if in_dtype == torch.bfloat16:
        x = synth.round_bf16(x)
    elif in_dtype == torch.float16:
        x = x.astype(np.float16).astype(np.float32)
    xd = torch.from_numpy(x).to("cuda", in_dtype)
    # significand bits of the output type: one rounding of the exact rotation
    ulp_half = {torch.float32: 2.0 ** -24, torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}[out_dtype]
    for inverse in (False, True):
        if out_dtype == in_dtype:
            y = xd.clone()
            opr.opr_rope(y, lay.pos_id, 1e6, inverse=inverse)
        else:
            y = torch.empty(xd.shape, dtype=out_dtype, device="cuda")
            opr.opr_rope(xd, lay.pos_id, 1e6, inverse=inverse, out=y, dev_status=lay.dev_status)
        ref = orc.rope(x, ref_lay.pos_id, 1e6, inverse=inverse)
        got = y.float().cpu().numpy()
        # fp32 arithmetic of the rotation adds a few 1e-7 on top of the final rounding
        assert np.all(np.abs(got - ref) <= np.abs(ref) * ulp_half + 2e-6)
    torch.cuda.synchronize()
    assert opr.read_status(lay.dev_status) == []


@pytest.mark.parametrize("d,offset", [(40, 0), (128, 1)])
def test_rope_general_form(d, offset):
    """Shapes the vectorised kernel does not take: d/2 not a multiple of 8, or a tensor off 16-byte alignment."""
    w = synth.make_workload(1)
    ref_lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    lay = opr.opr_build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    rng = np.random.default_rng(1)
    x = synth.round_bf16(rng.standard_normal((lay.total, 3, d)).astype(np.float32))
    buf = torch.empty(x.size + offset, dtype=torch.bfloat16, device="cuda")
    xd = buf[offset:].view(x.shape)
    xd.copy_(torch.from_numpy(x).to("cuda", torch.bfloat16))
    assert (xd.data_ptr() % 16 != 0) == (offset != 0)
    opr.opr_rope(xd, lay.pos_id, 1e6)
    ref = orc.rope(x, ref_lay.pos_id, 1e6)
    got = xd.float().cpu().numpy()
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 2e-6)


def test_rope_fp16_overflow_is_flagged():
    lay = opr.opr_build_layout([[4, 0, 0]], [0, 1], [0, 1])
    x = torch.full((4, 1, 64), 1e5, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(x.shape, dtype=torch.float16, device="cuda")
    opr.opr_rope(x, lay.pos_id, 1e4, out=y, dev_status=lay.dev_status)
    torch.cuda.synchronize()
    assert _abi.DEV_BITS[16] in opr.read_status(lay.dev_status)


def test_rope_binding_rejects_bad_positions():
    """pos_id must be int32 with one entry per row: the kernel reads pos_id[t] for every row t."""
    lay = opr.opr_build_layout([[4, 0, 0]], [0, 1], [0, 1])
    x = torch.zeros((4, 1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(opr.OprError):
        opr.opr_rope(x, lay.pos_id.long(), 1e4)
    with pytest.raises(opr.OprError):
        opr.opr_rope(x, lay.pos_id[:3], 1e4)


@pytest.mark.parametrize("shape", [(1000, 3, 64), (1001, 3, 2)])  # 16-byte vector form; element form
@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32])
def test_rope_without_positions_is_a_type_conversion(in_dtype, shape):
    """pos_id NULL: no rotation, the value rounded once to the output type (the fp16 copy of v
    that the forward's P V product takes): bit for bit torch's round-to-nearest conversion;
    a value beyond the fp16 range is flagged."""
    rng = np.random.default_rng(7)
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * 100).to("cuda", in_dtype)
    y = torch.empty(x.shape, dtype=torch.float16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    opr.opr_rope(x, None, 1e4, out=y, dev_status=st)
    torch.cuda.synchronize()
    assert opr.read_status(st) == []
    assert torch.equal(y.view(torch.int16), x.to(torch.float16).view(torch.int16))
    x[17, 1, 1] = 1e5
    opr.opr_rope(x, None, 1e4, out=y, dev_status=st)
    torch.cuda.synchronize()
    assert _abi.DEV_BITS[16] in opr.read_status(st)

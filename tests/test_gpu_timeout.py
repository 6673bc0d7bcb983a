"""The bounded-wait timeout path of the attention kernels, taken on purpose.

Every pipeline wait in the kernels (a TMA copy, a tensor-core product, another
warp's hand-off) has a time limit.  The test hook of include/opr_testing.h sets
that limit to 0, so a wait whose phase has not completed at its first test
gives up: the block stops issuing work, lets its copies and products in flight
finish, frees its tensor memory, returns, and reports OPR_DEV_WAIT_TIMEOUT.
Afterwards a normal call in the same process must still match the oracle: the
context stays usable.  Nothing here faults, traps or hangs a GPU.
"""

import numpy as np
import pytest
import torch

import block_sparse_masked_segment_b200 as opr
import synth
from oracle import opr_oracle as orc
from parity_helpers import assert_close, inputs, to_dev

pytestmark = pytest.mark.gpu

TIMEOUT = "pipeline wait timeout"


@pytest.mark.parametrize("kind", ["single head", "head pair"])
def test_wait_timeout_is_reported_and_the_context_stays_usable(kind):
    if kind == "single head":
        w = synth.make_workload(0)  # 160 tokens, one head: the one-head forward kernel
    else:
        w = synth.random_small_workload(9, n_seqs=1, max_convs=2, max_turns=2, hq=4, hkv=2, d=128, base=1e6)
    lib = opr.load_library()
    q, k, v, do = inputs(w, 90)
    att = opr.OnePassAttention(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, base=w.base)
    qd, kd, vd, dod = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    torch.cuda.synchronize()
    assert opr.read_status(att.layout.dev_status) == []
    prev = lib.opr_testing_set_wait_limit_ns(0)
    try:
        o, lse, qr, kr = att.forward(qd, kd, vd)
        torch.cuda.synchronize()
        fwd_status = opr.read_status(att.layout.dev_status)
        att.layout.dev_status.zero_()
        att.backward(qr, kr, vd, o, dod, lse)
        torch.cuda.synchronize()
        bwd_status = opr.read_status(att.layout.dev_status)
    finally:
        lib.opr_testing_set_wait_limit_ns(prev)
    assert fwd_status == [TIMEOUT]
    assert bwd_status == [TIMEOUT]
    # the same calls with the default limit: no status bit, and the oracle's values
    att.layout.dev_status.zero_()
    o, lse, qr, kr = att.forward(qd, kd, vd)
    dq, dk, dv = att.backward(qr, kr, vd, o, dod, lse)
    torch.cuda.synchronize()
    assert opr.read_status(att.layout.dev_status) == []
    lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
    ro, rlse = orc.forward(q, k, v, lay, w.base)
    rdq, rdk, rdv = orc.backward(q, k, v, ro, do, rlse, lay, w.base)
    for name, g, r in (("O", o, ro), ("LSE", lse, rlse), ("dQ", dq, rdq), ("dK", dk, rdk), ("dV", dv, rdv)):
        assert_close(name, g.float().cpu().numpy(), r)

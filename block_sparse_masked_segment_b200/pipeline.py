"""The one-pass attention layer as a sequence of library calls.

forward:  opr_rope(q), opr_rope(k) by the layout's position ids (bf16 in,
          fp16 out) -> opr_attn_fwd
backward: opr_attn_bwd with the position ids, which rotates dq and dk back
          (the gradients w.r.t. the unrotated q and k)
(One-Pass to Reason: positions from "位置 ID 策略", mask from "分块稀疏注意力掩码").
Every numerical step runs in libopr's CUDA kernels; this module only orders the
calls and keeps buffers.
"""

from __future__ import annotations

import numpy as np
import torch

from ._abi import Layout, opr_attn_bwd, opr_attn_fwd, opr_build_layout, opr_rope


def visible_pairs_closed_form(turn_lens, conv_turn_ptr) -> int:
    """Visible (q, k) pairs per head of a one-pass layout, counted per turn.

    With A_i = sum_{j<i}(h_j + r_j) (the history length seen by turn i):
    h rows see A_i + causal h; t rows A_i + h + causal t; r^in rows A_i + h +
    causal r; r^out rows A_i + h + t + causal r.  Used as the useful-work
    count of the throughput metric (the pages' complexity analysis counts the
    same attended pairs).
    """
    tl = np.asarray(turn_lens, dtype=np.int64).reshape(-1, 3)
    cp = np.asarray(conv_turn_ptr, dtype=np.int64)
    total = 0
    for c in range(len(cp) - 1):
        A = 0
        for h, t, r in tl[cp[c]:cp[c + 1]]:
            total += h * A + h * (h + 1) // 2
            total += t * (A + h) + t * (t + 1) // 2
            total += r * (A + h) + r * (r + 1) // 2
            total += r * (A + h + t) + r * (r + 1) // 2
            A += h + r
    return int(total)


def useful_flops(pairs: int, hq: int, d: int, backward: bool) -> float:
    """4 d flops per visible pair and q head forward; 2.5 times that backward."""
    f = 4.0 * d * pairs * hq
    return f * 3.5 if backward else f


def one_pass_forward(q_pre, k_pre, v, lay: Layout, base: float, scale=None, out_dtype=torch.float32):
    """RoPE (bf16 in, fp16 out), an fp16 copy of v (so that P V runs with fp16 P), all three
    written in the layout's attention order, then masked attention.  Returns (o, lse, q_rot,
    k_rot): o and lse in the stream order, q_rot and k_rot in the attention order (the form
    one_pass_backward takes)."""
    q = torch.empty(q_pre.shape, dtype=torch.float16, device=q_pre.device)
    k = torch.empty(k_pre.shape, dtype=torch.float16, device=k_pre.device)
    v16 = torch.empty(v.shape, dtype=torch.float16, device=v.device)
    # rotated q, k and the fp16 v go to the attention order (rows lay.attn_pos)
    opr_rope(q_pre, lay.pos_id, base, out=q, dev_status=lay.dev_status, row_map=lay.attn_pos)
    opr_rope(k_pre, lay.pos_id, base, out=k, dev_status=lay.dev_status, row_map=lay.attn_pos)
    opr_rope(v, None, base, out=v16, dev_status=lay.dev_status, row_map=lay.attn_pos)
    o, lse = opr_attn_fwd(q, k, v16, lay, scale, out_dtype)
    return o, lse, q, k


def one_pass_backward(q_rot, k_rot, v, o, do, lse, lay: Layout, base: float, scale=None):
    """Gradients w.r.t. the unrotated q, k and v (the backward rotates dq and dk back)."""
    return opr_attn_bwd(q_rot, k_rot, v, o, do, lse, lay, scale, rope_base=base)


class OnePassAttention:
    """Layout built once from per-turn lengths, then forward/backward calls.

    >>> att = OnePassAttention(turn_lens, conv_turn_ptr, seq_conv_ptr, base=1e6)
    >>> o, lse, q_rot, k_rot = att.forward(q, k, v)
    >>> dq, dk, dv = att.backward(q_rot, k_rot, v, o, do, lse)
    """

    def __init__(self, turn_lens, conv_turn_ptr, seq_conv_ptr, base: float, device="cuda"):
        self.layout = opr_build_layout(turn_lens, conv_turn_ptr, seq_conv_ptr, device=device)
        self.base = base

    def forward(self, q_pre, k_pre, v, scale=None, out_dtype=torch.float32):
        return one_pass_forward(q_pre, k_pre, v, self.layout, self.base, scale, out_dtype)

    def backward(self, q_rot, k_rot, v, o, do, lse, scale=None):
        return one_pass_backward(q_rot, k_rot, v, o, do, lse, self.layout, self.base, scale)

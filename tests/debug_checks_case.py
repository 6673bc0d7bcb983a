"""One forward + backward of the small workload (index 0) through whichever library the
binding loaded, on a consistent layout and on layouts with one table entry made out of
range on purpose.  tests/test_gpu_debug_checks.py runs it in-process with the release
library and as a child process with OPR_DEBUG_CHECKS=1 (the bounds-checking library).

Run as a script: ``python tests/debug_checks_case.py OUT.npz`` writes the clean run's
outputs and the status words of the corrupted runs.  Only the debug library is ever given
a corrupted layout: its kernels check the tile tables before any access they steer.
"""

from __future__ import annotations

import dataclasses
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import block_sparse_masked_segment_b200 as opr  # noqa: E402
import synth  # noqa: E402

CORRUPTIONS = ("row_cnt", "row_entry", "col_cnt", "col_entry", "cu_seqlens")


def inputs():
    w = synth.make_workload(0)
    rng = np.random.default_rng(2024)
    n = w.total_tokens
    q, k, v, do = (synth.gaussian(rng, (n, h, w.d)) for h in (w.hq, w.hkv, w.hkv, w.hq))
    dev = lambda x: torch.from_numpy(x).to("cuda:0", torch.bfloat16)  # noqa: E731
    return w, dev(q), dev(k), dev(v), dev(do)


def run(lay, w, q, k, v, do):
    """Rope, forward, backward; returns (outputs, fwd status bits, bwd status bits)."""
    qr = torch.empty(q.shape, dtype=torch.float16, device=q.device)
    kr = torch.empty(k.shape, dtype=torch.float16, device=q.device)
    va = torch.empty(v.shape, dtype=torch.bfloat16, device=q.device)
    # the attention calls take q, k and v in the layout's attention order
    opr.opr_rope(q, lay.pos_id, w.base, out=qr, row_map=lay.attn_pos)
    opr.opr_rope(k, lay.pos_id, w.base, out=kr, row_map=lay.attn_pos)
    opr.opr_rope(v, None, w.base, out=va, row_map=lay.attn_pos)
    lay.dev_status.zero_()
    o, lse = opr.opr_attn_fwd(qr, kr, va, lay, out_dtype=torch.bfloat16)
    fwd_bits = int(lay.dev_status.item())
    lay.dev_status.zero_()
    dq, dk, dv = opr.opr_attn_bwd(qr, kr, v, o, do, lse, lay)
    bwd_bits = int(lay.dev_status.item())
    outs = {"o": o.float().cpu().numpy(), "lse": lse.cpu().numpy(), "dq": dq.cpu().numpy(),
            "dk": dk.cpu().numpy(), "dv": dv.cpu().numpy()}
    return outs, fwd_bits, bwd_bits


def corrupted(lay, kind: str):
    """A copy of the layout with one out-of-range table value (tile 0 of sequence 0)."""
    bad = dataclasses.replace(lay, workspace=lay.workspace.clone(), cu_seqlens=lay.cu_seqlens.clone(),
                              dev_status=torch.zeros_like(lay.dev_status))
    off = opr.layout_table_offsets(bad)
    ws32 = bad.workspace.view(torch.int32)
    T = bad.T
    if kind == "row_cnt":
        ws32[off["row_cnt"] // 4] = T + 1  # more entries than a row list holds
    elif kind == "row_entry":
        ws32[off["row_list"] // 4] = ((T + 2) << 4) | 1  # a key tile past the sequence
    elif kind == "col_cnt":
        ws32[off["col_cnt"] // 4] = T + 1
    elif kind == "col_entry":
        ws32[off["col_list"] // 4] = ((T + 2) << 4) | 1
    elif kind == "cu_seqlens":
        bad.cu_seqlens[-1] = bad.total + 1000  # last sequence ends past the tokens
    else:
        raise ValueError(kind)
    return bad


def main(out_path: str) -> None:
    assert opr.opr_version().endswith("debug-checks"), "corrupted layouts go to the debug library only"
    torch.cuda.set_device(0)
    w, q, k, v, do = inputs()
    lay = opr.opr_build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, device="cuda:0")
    outs, fb, bb = run(lay, w, q, k, v, do)
    result = {f"clean_{name}": a for name, a in outs.items()}
    result["clean_bits"] = np.array([fb, bb])
    for kind in CORRUPTIONS:
        _, fb, bb = run(corrupted(lay, kind), w, q, k, v, do)
        result[f"bits_{kind}"] = np.array([fb, bb])
    torch.cuda.synchronize()
    np.savez(out_path, **result)


if __name__ == "__main__":
    main(sys.argv[1])

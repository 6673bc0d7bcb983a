"""The bounds-checking library (libopr_debug.so, built with OPR_DEBUG_CHECKS) on a B200.

- On a consistent layout it computes what the release library computes, bit for bit, and
  leaves the status word clean.
- On a layout whose tile tables carry one out-of-range value (a count longer than a tile
  list, a list entry past the sequence, a sequence bound past the tokens) the attention
  kernels that read that table set OPR_DEV_BOUNDS (32) instead of using the value; the
  kernels that do not read it stay clean.

The debug library runs in a child process (the binding picks the library when it is
imported).  Only the debug library ever sees a corrupted layout: its kernels check the
tables before the first access they steer, so no out-of-range access is made.
"""

import os
import subprocess
import sys

import numpy as np
import pytest

from block_sparse_masked_segment_b200 import build as opr_build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BOUNDS = 32


@pytest.fixture(scope="module")
def debug_run(tmp_path_factory):
    opr_build.build(debug=True)
    out = tmp_path_factory.mktemp("debug_checks") / "debug.npz"
    env = dict(os.environ, OPR_DEBUG_CHECKS="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_checks_case.py"), str(out)],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    return dict(np.load(out))


def test_debug_library_matches_release_bit_for_bit(debug_run):
    import torch

    import block_sparse_masked_segment_b200 as opr
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import debug_checks_case as case

    assert not opr.opr_version().endswith("debug-checks")
    torch.cuda.set_device(0)
    w, q, k, v, do = case.inputs()
    lay = opr.opr_build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, device="cuda:0")
    outs, fb, bb = case.run(lay, w, q, k, v, do)
    assert (fb, bb) == (0, 0)
    assert list(debug_run["clean_bits"]) == [0, 0]
    for name, a in outs.items():
        np.testing.assert_array_equal(debug_run[f"clean_{name}"], a, err_msg=name)


@pytest.mark.parametrize("kind,fwd_hit,bwd_hit", [
    ("row_cnt", True, True),      # forward and dQ kernels read the row tables
    ("row_entry", True, True),
    ("col_cnt", False, True),     # only the dK/dV kernel reads the column tables
    ("col_entry", False, True),
    ("cu_seqlens", True, True),   # every attention kernel and the row terms read it
])
def test_out_of_range_table_value_sets_bounds_bit(debug_run, kind, fwd_hit, bwd_hit):
    fb, bb = (int(x) for x in debug_run[f"bits_{kind}"])
    assert bool(fb & BOUNDS) == fwd_hit, (kind, fb)
    assert bool(bb & BOUNDS) == bwd_hit, (kind, bb)
    # nothing else went wrong: no other status bit, in particular no wait timeout
    assert fb & ~BOUNDS == 0 and bb & ~BOUNDS == 0, (kind, fb, bb)

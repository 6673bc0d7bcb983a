"""The C-ABI library without a GPU: it loads, exports every entry point that
include/opr.h declares, and rejects bad arguments on the host before touching
the device."""

import ctypes
import os
import re

import numpy as np
import pytest

import block_sparse_masked_segment_b200 as opr
from block_sparse_masked_segment_b200 import build as opr_build
from block_sparse_masked_segment_b200.pipeline import visible_pairs_closed_form
import synth
from oracle import opr_oracle as orc

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


@pytest.fixture(scope="module")
def lib():
    opr_build.build()
    return opr.load_library()


def declared_symbols():
    """Every entry point that a header under include/ declares."""
    text = "".join(open(os.path.join(INCLUDE, f)).read() for f in sorted(os.listdir(INCLUDE)) if f.endswith(".h"))
    return sorted(set(re.findall(r"OPR_API\s+[\w\s\*]+?\b(opr_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 8
    assert set(names) == set(opr.EXPORTED_SYMBOLS)
    for name in names:
        assert hasattr(lib, name), name


def test_version(lib):
    assert opr.opr_version().startswith("opr ")


def test_wait_limit_hook_round_trips(lib):
    """The test hook of include/opr_testing.h sets the pipeline-wait limit and returns the old one
    (host code only: no kernel runs)."""
    prev = lib.opr_testing_set_wait_limit_ns(12345)
    assert prev == 2_000_000_000
    assert lib.opr_testing_set_wait_limit_ns(prev) == 12345


def test_layout_tables_hook(lib):
    """Offsets of the tile tables inside the layout workspace: in order, non-overlapping, inside it."""
    n_seqs, n_convs, n_turns, total, max_seqlen = 2, 5, 20, 30000, 16384
    out = (ctypes.c_uint64 * 4)()
    assert lib.opr_testing_layout_tables(n_seqs, n_convs, n_turns, total, max_seqlen,
                                         ctypes.cast(out, ctypes.c_void_p)) == 0
    T = (max_seqlen + 127) // 128
    n_tiles = n_seqs * T
    row_cnt, row_list, col_cnt, col_list = (int(x) for x in out)
    assert row_list - row_cnt >= 4 * n_tiles and col_cnt - row_list >= 4 * n_tiles * T
    assert col_list - col_cnt >= 4 * n_tiles
    assert col_list + 4 * n_tiles * T <= opr.opr_layout_workspace_bytes(n_seqs, n_convs, n_turns, total, max_seqlen)
    assert lib.opr_testing_layout_tables(-1, n_convs, n_turns, total, max_seqlen, ctypes.cast(out, ctypes.c_void_p)) == 1
    assert lib.opr_testing_layout_tables(n_seqs, n_convs, n_turns, total, max_seqlen, None) == 1


def test_debug_library_builds_and_exports_the_same_symbols(lib):
    """The bounds-checking build (OPR_DEBUG_CHECKS) has every entry point and says so in its version."""
    path = opr_build.build(debug=True)
    assert path.endswith("libopr_debug.so")
    dbg = ctypes.CDLL(path)
    for name in declared_symbols():
        assert hasattr(dbg, name), name
    dbg.opr_version.restype = ctypes.c_char_p
    assert dbg.opr_version().decode().endswith("debug-checks")
    assert not opr.opr_version().endswith("debug-checks")


def test_binding_loads_the_debug_library_on_request(lib):
    """OPR_DEBUG_CHECKS=1 in the environment points the binding at libopr_debug.so."""
    import subprocess
    import sys
    opr_build.build(debug=True)
    root = os.path.dirname(INCLUDE)
    code = "import block_sparse_masked_segment_b200 as o; o.load_library(); print(o.library_path()); print(o.opr_version())"
    env = dict(os.environ, OPR_DEBUG_CHECKS="1")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    path, version = r.stdout.split("\n")[:2]
    assert path.endswith("libopr_debug.so") and version.endswith("debug-checks")


def test_workspace_queries(lib):
    b = opr.opr_layout_workspace_bytes(2, 5, 20, 30000, 16384)
    assert b > 4 * 30000 and b % 256 == 0
    assert opr.opr_layout_workspace_bytes(-1, 5, 20, 30000, 16384) == 0
    assert opr.opr_layout_workspace_bytes(1, 1, 1, 1 << 31, 100) == 0
    assert opr.opr_attn_bwd_workspace_bytes(2, 1000, 8, 128) >= 2 * 4 * 8 * 2 * 8 * 128


def test_host_argument_checks(lib):
    """Null pointers, bad head counts and dims are refused with OPR_INVALID_ARG
    (1) before any CUDA call, so this runs without a GPU."""
    N = None
    # opr_build_layout with null outputs
    assert lib.opr_build_layout(N, N, N, 1, 1, 1, 10, 10, N, N, N, N, N, N, N, N, 0, N, N) == 1
    # negative sizes
    assert lib.opr_build_layout(N, N, N, -1, 1, 1, 10, 10, N, N, N, N, N, N, N, N, 0, N, N) == 1
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the checks fail first
    # opr_rope: odd head_dim, bad dtype, null pointer, in place with two types
    assert lib.opr_rope(N, 0, N, 0, N, N, 10, 2, 63, 1e4, 0, N, N) == 1
    assert lib.opr_rope(N, 7, N, 0, N, N, 10, 2, 64, 1e4, 0, N, N) == 2
    assert lib.opr_rope(N, 0, N, 0, N, N, 10, 2, 64, 1e4, 0, N, N) == 1
    assert lib.opr_rope(fake, 0, fake, 2, fake, N, 10, 2, 64, 1e4, 0, N, N) == 1
    # a row map writes rows elsewhere, so it cannot work in place
    assert lib.opr_rope(fake, 0, fake, 0, fake, fake, 10, 2, 64, 1e4, 0, N, N) == 1
    # opr_attn_fwd: null q; hq % hkv != 0; head_dim 96
    assert lib.opr_attn_fwd(N, fake, fake, 2, 0, fake, fake, fake, 1, 1, 1, 100, 100, 4, 2, 128, 0.1,
                            fake, 0, fake, fake, N) == 1
    assert lib.opr_attn_fwd(fake, fake, fake, 2, 0, fake, fake, fake, 1, 1, 1, 100, 100, 6, 4, 128, 0.1,
                            fake, 0, fake, fake, N) == 1
    assert lib.opr_attn_fwd(fake, fake, fake, 2, 0, fake, fake, fake, 1, 1, 1, 100, 100, 4, 2, 96, 0.1,
                            fake, 0, fake, fake, N) == 1
    # v of fp32 is not an MMA type (fp16 or bf16 only)
    assert lib.opr_attn_fwd(fake, fake, fake, 2, 1, fake, fake, fake, 1, 1, 1, 100, 100, 4, 2, 128, 0.1,
                            fake, 0, fake, fake, N) == 2
    # q/k of fp32 are not an MMA type
    assert lib.opr_attn_fwd(fake, fake, fake, 1, 0, fake, fake, fake, 1, 1, 1, 100, 100, 4, 2, 128, 0.1,
                            fake, 0, fake, fake, N) == 2
    # opr_attn_bwd_stages: unknown stage bits
    assert lib.opr_attn_bwd_stages(fake, fake, fake, 2, fake, 0, fake, fake, fake, fake, fake, 1, 1, 1, 100, 100,
                                   4, 2, 128, 0.1, fake, fake, fake, N, 0.0, fake, 1 << 20, fake, 8, N) == 1
    # a rotary position array without a valid base
    assert lib.opr_attn_bwd(fake, fake, fake, 2, fake, 0, fake, fake, fake, fake, fake, 1, 1, 1, 100, 100,
                            4, 2, 128, 0.1, fake, fake, fake, fake, 0.5, fake, 1 << 30, fake, N) == 1
    # q/k in bf16 are refused: the attention calls take the rotated q and k in fp16 only
    assert lib.opr_attn_fwd(fake, fake, fake, 0, 0, fake, fake, fake, 1, 1, 1, 100, 100, 4, 2, 128, 0.1,
                            fake, 0, fake, fake, N) == 2
    assert lib.opr_attn_bwd(fake, fake, fake, 0, fake, 0, fake, fake, fake, fake, fake, 1, 1, 1, 100, 100,
                            4, 2, 128, 0.1, fake, fake, fake, N, 0.0, fake, 1 << 30, fake, N) == 2
    # more tokens than n_seqs * ceil(max_seqlen / 128) * 128 (the bound every workspace is sized
    # by): refused on the host, by every call that sizes buffers from (n_seqs, max_seqlen)
    assert lib.opr_attn_fwd(fake, fake, fake, 2, 0, fake, fake, fake, 1, 1, 1, 300, 100, 4, 2, 128, 0.1,
                            fake, 0, fake, fake, N) == 1
    assert lib.opr_attn_bwd(fake, fake, fake, 2, fake, 0, fake, fake, fake, fake, fake, 1, 1, 1, 300, 100,
                            4, 2, 128, 0.1, fake, fake, fake, N, 0.0, fake, 1 << 30, fake, N) == 1
    assert lib.opr_attn_bwd_noalloc(fake, fake, fake, 2, fake, 0, fake, fake, fake, fake, fake, 1, 1, 1, 300, 100,
                                    4, 2, 128, 0.1, fake, fake, fake, N, 0.0, fake, N) == 1
    assert lib.opr_build_layout(fake, fake, fake, 1, 1, 1, 300, 100, fake, fake, fake, fake, fake, fake, fake, fake,
                                1 << 30, fake, N) == 1
    assert opr.opr_layout_workspace_bytes(1, 1, 1, 300, 100) == 0
    # empty problems are no-ops
    assert lib.opr_attn_fwd(N, N, N, 2, 0, N, N, N, 0, 0, 0, 0, 0, 4, 2, 128, 0.1, N, 0, N, N, N) == 0


def test_closed_form_pair_count_matches_oracle():
    """The benchmark's useful-work count equals the oracle's mask count."""
    for seed in range(4):
        w = synth.random_small_workload(seed)
        lay = orc.build_layout(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr)
        assert visible_pairs_closed_form(w.turn_lens, w.conv_turn_ptr) == orc.visible_pairs(lay)


def test_npass_workload_is_causal_sequences():
    w = synth.make_workload(3, n_turns=4)
    nw, origin = synth.npass_workload(w)
    assert nw.n_seqs == 4 and [i for _, i in origin] == [0, 1, 2, 3]
    # N-pass sequence of turn i: sum_{j<i}(h+r) + h + t + r = 384 i + 896
    np.testing.assert_array_equal(nw.seq_lengths(), [896, 1280, 1664, 2048])


def test_duplication_entry_points_check_arguments_on_the_host():
    """Host-side checks return before any device work (fake pointers are never touched)."""
    lib = opr.load_library()
    fake = ctypes.c_void_p(1 << 20)
    # negative sizes, a null status word, more original tokens than one-pass tokens
    assert lib.opr_duplication_index(fake, fake, 1, -1, 10, 5, fake, fake, fake, None) == 1
    assert lib.opr_duplication_index(fake, fake, 1, 2, 10, 5, fake, fake, None, None) == 1
    assert lib.opr_duplication_index(fake, fake, 1, 2, 10, 11, fake, fake, fake, None) == 1
    assert lib.opr_gather_rows(fake, 5, 0, fake, 10, fake, None, None) == 1
    assert lib.opr_gather_rows(None, 5, 16, fake, 10, fake, None, None) == 1
    assert lib.opr_gather_rows(fake, 5, 16, fake, 0, fake, None, None) == 0  # nothing to copy
    assert lib.opr_fold_rows(fake, 10, 0, fake, 2, 5, fake, None, None) == 1
    assert lib.opr_fold_rows(fake, 10, 4, fake, 0, 5, fake, None, None) == 1  # no slots
    assert lib.opr_fold_rows(fake, 10, 4, fake, 2, 0, fake, None, None) == 0
    ws = lib.opr_kpass_index_workspace_bytes(10, 20)
    assert ws >= 8 * (11 + 21)
    assert lib.opr_kpass_index(fake, 10, fake, fake, 20, 100, 50, 3, fake, fake, fake, ws - 256, fake, None) == 4
    assert lib.opr_kpass_plan(fake, fake, fake, 1, 1, 2, 0, 2, 1, fake, fake, fake, fake, fake, None) == 1  # K = 0


def _kpass_sizes(lib, w, K):
    lens = np.ascontiguousarray(np.asarray(w.turn_lens, dtype=np.int32).reshape(-1))
    cp = np.ascontiguousarray(np.asarray(w.conv_turn_ptr, dtype=np.int32))
    sp = np.ascontiguousarray(np.asarray(w.seq_conv_ptr, dtype=np.int32))
    out = [ctypes.c_int64(-1) for _ in range(5)]
    st = lib.opr_kpass_sizes(lens.ctypes.data, cp.ctypes.data, sp.ctypes.data, sp.size - 1, cp.size - 1,
                             lens.size // 3, K, *(ctypes.byref(x) for x in out))
    return st, [x.value for x in out]


@pytest.mark.parametrize("K", [1, 2, 3, 5])
def test_kpass_sizes_match_the_oracle(K):
    """opr_kpass_sizes is host code: every size it reports (turns, passes, tokens, longest
    sequence, original tokens) is checked against the oracle's arrangement without a GPU."""
    lib = opr.load_library()
    for seed in (21, 22):
        w = synth.random_small_workload(seed, n_seqs=3, max_convs=4, max_turns=6)
        st, (nt, nc, total, max_seqlen, orig) = _kpass_sizes(lib, w, K)
        assert st == 0
        l2, c2, s2, _ = orc.kpass_plan(w.turn_lens, w.conv_turn_ptr, w.seq_conv_ptr, K)
        lay = orc.build_layout(l2, c2, s2)
        assert (nt, nc) == (len(l2), len(c2) - 1)
        assert total == int(lay.cu_seqlens[-1])
        assert max_seqlen == int(np.diff(lay.cu_seqlens).max())
        assert orig == int(np.asarray(w.turn_lens, dtype=np.int64).sum())
    # bad input: K = 0, a negative length, pointers that do not span the turns
    assert _kpass_sizes(lib, w, 0)[0] == 1
    bad = synth.make_custom_workload([[[(1, -2, 3)]]], hq=1, hkv=1, d=64, base=1e4)
    assert _kpass_sizes(lib, bad, 2)[0] == 1


def test_loss_row_count_matches_the_oracle():
    """opr_loss_row_count is host code: checked against the oracle's loss rows without a GPU."""
    import synth
    from oracle import opr_oracle as orc

    lib = opr.load_library()
    for seed in range(4):
        w = synth.random_small_workload(seed, max_turns=6)
        lens = np.ascontiguousarray(np.asarray(w.turn_lens, dtype=np.int32).reshape(-1, 3))
        rows, _ = orc.loss_rows(w.turn_lens, w.conv_turn_ptr)
        assert lib.opr_loss_row_count(lens.ctypes.data, lens.shape[0]) == len(rows)
    bad = np.asarray([[1, -2, 3]], dtype=np.int32)
    assert lib.opr_loss_row_count(bad.ctypes.data, 1) == -1

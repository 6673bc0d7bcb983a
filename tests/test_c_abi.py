"""The C ABI from plain C: tests/c/host_calls.c includes opr.h, is compiled with gcc -std=c99
-pedantic-errors and linked against lib/libopr.so, and calls the host-only entry points."""

import os
import shutil
import subprocess

import pytest

import block_sparse_masked_segment_b200 as opr
from oracle import opr_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_c99_and_host_calls_work():
    lib = opr.library_path()
    out_dir = os.path.join(ROOT, ".pytest_cache", "c_abi")  # git-ignored, inside the repository
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "host_calls")
    cuda_inc = "/usr/local/cuda/include"
    cc = ["gcc", "-std=c99", "-pedantic-errors", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
          "-I", cuda_inc, os.path.join(ROOT, "tests", "c", "host_calls.c"), lib, "-o", str(exe),
          f"-Wl,-rpath,{os.path.dirname(lib)}"]
    out = subprocess.run(cc, capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    lines = run.stdout.split()
    assert lines[0] == "opr"
    turns = [[2, 3, 2], [1, 2, 1], [4, 2, 3]]
    l2, c2, s2, _ = orc.kpass_plan(turns, [0, 2, 3], [0, 2], 2)
    lay = orc.build_layout(l2, c2, s2)
    rows, _ = orc.loss_rows(turns, [0, 2, 3])
    vals = [int(x) for x in lines[-8:]]
    total = int(lay.cu_seqlens[-1])
    assert vals == [len(l2), len(c2) - 1, total, total, 20, len(rows), 1, 1]

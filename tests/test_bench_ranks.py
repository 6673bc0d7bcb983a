"""The N>1 path of bench.py on CPU: two gloo ranks, each with its own batch.

bench.py scales weakly: every rank runs the whole path on a batch of its own
(drawn from a rank-specific seed, same configuration), the job's time is the
maximum of the ranks' times and its work the sum of their work.  These tests
run that plumbing as two real processes over gloo; only the device is the CPU.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        ranks = bench.Ranks(world, torch.device("cpu"))
        ranks.barrier()
        # a rank's "step time" and "work": the job takes the slowest rank's time and all ranks' work
        t_ms = 10.0 + 5.0 * rank
        work = 100.0 * (rank + 1)
        job_ms = ranks.max(t_ms)
        job_work = ranks.sum(work)
        w = bench.rank_workload(1, rank)
        ranks.barrier()
        out.put((rank, job_ms, job_work, w.total_tokens, w.hq, w.hkv, w.d, np.asarray(w.turn_lens).ravel().tolist()))
    except Exception as e:  # surface the failure to the parent instead of a queue timeout
        out.put((rank, "error", repr(e)))
        raise
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_time_by_max_and_work_by_sum():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r = out.get(timeout=120)
        assert r[1] != "error", r
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        _, job_ms, job_work, *_ = res[rank]
        assert job_ms == pytest.approx(15.0)  # max over ranks, identical on every rank
        assert job_work == pytest.approx(300.0)  # sum over ranks
    # same configuration shape on both ranks, different batches (weak scaling)
    a, b = res[0], res[1]
    assert a[4:7] == b[4:7]
    assert a[7] != b[7]


def test_rank_workload_matches_the_single_gpu_workload_on_rank_0():
    w0 = bench.rank_workload(1, 0)
    w = synth.make_workload(1, seed=1000 + 1)
    assert w0.total_tokens == w.total_tokens
    assert np.array_equal(np.asarray(w0.turn_lens), np.asarray(w.turn_lens))


def test_single_rank_reductions_are_identity():
    ranks = bench.Ranks(1, torch.device("cpu"))
    ranks.barrier()
    assert ranks.max(3.5) == 3.5
    assert ranks.sum(2.0) == 2.0

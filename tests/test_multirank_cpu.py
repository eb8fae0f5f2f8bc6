"""The multi-rank path of bench.py on the CPU: two gloo ranks (127.0.0.1).

Each GPU rank of `bench.py --gpus N` times its own independent batch; the
only cross-rank steps are the barriers and the maximum of the per-rank
timings, and the reported value is every rank's units over the slowest
rank's time.  These tests run those steps with world_size 2 on gloo.
"""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from graph_transformer_sparse_kmip_b200 import workloads as wl

        got_ws, got_rank, got_local = bench._dist()
        dist.barrier()
        # Rank r took (2 + r) ms forward and (9 - 3 r) ms per step.
        t_fwd, t_tot = bench.max_over_ranks([2.0 + rank, 9.0 - 3 * rank], ws,
                                            torch.device("cpu"))
        q0 = bench.rank_inputs(wl.WORKLOADS["tiny_n1024_f32"], rank)["Q"]
        digest = float(q0.double().sum())
        ref = bench.run_reference(type("A", (), {"workload": "tiny_n1024_f32", "k": None,
                                                 "steps": 1, "warmup": 0})(), ws, rank) \
            if rank == 1 else "skipped"
        out[rank] = (got_ws, got_rank, got_local, t_fwd, t_tot, digest, ref)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True,
                           start_method="spawn")
        return dict(out)


def test_ranks_see_their_place(two_ranks):
    for r in (0, 1):
        ws, rank, local = two_ranks[r][:3]
        assert (ws, rank, local) == (2, r, r)


def test_timings_are_the_max_over_ranks(two_ranks):
    for r in (0, 1):
        t_fwd, t_tot = two_ranks[r][3:5]
        assert t_fwd == 3.0 and t_tot == 9.0


def test_ranks_draw_independent_batches(two_ranks):
    assert two_ranks[0][5] != two_ranks[1][5]


def test_reference_arm_runs_on_rank_zero_only(two_ranks):
    assert two_ranks[1][6] is None


def test_job_throughput_counts_every_rank():
    import bench
    assert bench.job_throughput(400000, 2, 10.0) == pytest.approx(8.0e7)
    assert bench.job_throughput(400000, 1, 10.0) == pytest.approx(4.0e7)
    assert bench.max_over_ranks([1.5, 2.5], 1, torch.device("cpu")) == [1.5, 2.5]

"""Host logic of the N > 1 benchmark path on CPU: two gloo ranks.

bench.py runs one independent stream per rank (replicas, no data-path
collective); the only cross-rank steps are the barrier around the timed
region and the max over ranks of the elapsed time.  These tests run those
steps with world size 2 over gloo, check that each rank draws its own
stream's inputs, and that the reference arm does no work off rank 0.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                          WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
        import datetime

        import bench
        import workloads
        dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
        got_ws, got_rank, got_local = bench.dist_env()
        elapsed = 10.0 + 5.0 * rank  # rank 1 is the slow one
        bench.barrier(ws)
        t_max = bench.max_over_ranks(elapsed, ws)
        rate = bench.whole_job_rate(21, ws, t_max)
        # replicas: each rank's stream has its own inputs
        w = workloads.WORKLOADS["tiny_fp32"]
        qx, _, _ = workloads.pass_inputs(w, rank, 0, 0)
        gathered = [torch.zeros_like(qx) for _ in range(ws)]
        dist.all_gather(gathered, qx)
        distinct = not torch.equal(gathered[0], gathered[1])
        # the reference arm returns without work on every rank but 0
        ref_rc = bench.run_reference(None, w) if rank != 0 else 0
        bench.barrier(ws)
        dist.destroy_process_group()
        q.put((rank, (got_ws, got_rank, got_local), t_max, rate, distinct, ref_rc))
    except Exception as e:  # reported to the parent
        q.put((rank, "error", repr(e)))


def test_two_gloo_ranks_barrier_max_and_replicas():
    ws = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(ws):
        item = q.get(timeout=180)
        results[item[0]] = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(ws):
        res = results[r]
        assert res[1] != "error", res
        _, env, t_max, rate, distinct, ref_rc = res
        assert env == (ws, r, r)
        assert t_max == pytest.approx(15.0)  # the slowest rank on every rank
        assert rate == pytest.approx(21 * ws / 0.015)
        assert distinct
        assert ref_rc == 0

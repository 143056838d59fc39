"""The N > 1 host path of bench.py on CPU: two ranks as spawned processes on
the gloo backend (no GPU).  Each rank runs its own replica; the job's time is
the maximum over ranks and its rate aggregates all ranks' units; the
reference arm runs on rank 0 only."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads as W
        bench.barrier(world)
        # per-rank step times: the slowest rank sets the job's time
        t = bench.max_over_ranks(1.0 + 0.5 * rank, world)
        rate = bench.aggregate_rate(100.0, t, world)
        # each rank draws its own replica (seed + rank)
        w = W.WORKLOADS["tiny"]
        case = W.make_case(w, seed=w.seed + rank, poison=False)
        q.put((rank, t, rate, float(case["q"].float().sum())))
    finally:
        dist.destroy_process_group()


def _run(world, target, *args):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q) + args) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


def test_two_ranks_time_is_the_max_and_rate_aggregates():
    res = _run(2, _worker)
    assert [r[1] for r in res] == [1.5, 1.5]
    assert all(r[2] == pytest.approx(2 * 100.0 / 1.5e-3) for r in res)
    assert res[0][3] != res[1][3]  # independent replicas


def _ref_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import contextlib
    import io
    import types
    import bench
    args = types.SimpleNamespace(workload="tiny", steps=1, warmup=0, gpus=world)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, world, rank)
    q.put((rank, buf.getvalue()))


def test_reference_arm_runs_on_rank_zero_only():
    res = _run(2, _ref_worker)
    import json
    line = json.loads(res[0][1].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert res[1][1] == ""

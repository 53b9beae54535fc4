"""bench.py's multi-rank plumbing on CPU: two gloo ranks (the launch a
`torchrun --nproc-per-node 2` would make) agree on the barrier, take the max of
their timed regions, and report whole-job throughput over both replicas."""
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


def _rank(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(world, backend="gloo")
    try:
        d.barrier()
        ms = 100.0 + 50.0 * rank  # rank 1 is the slow one
        m = d.max(ms)
        q.put((rank, d.world, m, bench.whole_job_rate(d.world, 64, m)))
    finally:
        d.close()


def test_two_gloo_ranks_max_and_whole_job_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    got = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, world, m, rate in got:
        assert world == 2
        assert m == 150.0  # max over ranks, on every rank
        assert rate == pytest.approx(2 * 64 / 0.150)


def test_single_rank_without_process_group():
    sys.path.insert(0, ROOT)
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    d = bench.Dist(1)
    assert d.world == 1 and d.pg is None and d.max(3.5) == 3.5
    d.barrier()
    d.close()
    with pytest.raises(SystemExit):
        bench.Dist(2)  # --gpus 2 without torchrun

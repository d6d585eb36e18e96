"""Host logic of bench.py's multi-GPU path, run as two gloo ranks on CPU:
the max-over-ranks timing, the whole-job throughput, and the reference arm
running on rank 0 only."""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    import io
    import contextlib
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank r took 10 * (r + 1) ms: every rank must see the slowest
        m = bench.max_over_ranks(10.0 * (rank + 1), dist, "cpu")
        v = bench.job_throughput(world, 4096 * 4096, 5, m)
        # the reference arm prints only on rank 0; other ranks do no work
        out = io.StringIO()
        if rank != 0:
            with contextlib.redirect_stdout(out):
                bench.run_reference(type("A", (), dict(workload="layer256_fp32", steps=1,
                                                       warmup=0))())
        dist.barrier()
        q.put((rank, m, v, out.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_as_the_slowest_and_count_all_work():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, v, out in res:
        assert m == 20.0
        assert v == pytest.approx(2 * 4096 * 4096 * 5 / 0.020)
        if rank != 0:
            assert out == ""


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.job_throughput(1, 100, 2, 1000.0) == 200.0

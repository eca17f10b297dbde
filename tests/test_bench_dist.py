"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (world size 2) exercise the
max-over-ranks timing reduction, the barriers around the timed region, the whole-job value (sum of
every rank's work over the slowest rank's time), and the reference arm's rank-0-only rule."""
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


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    ws, r = bench.init_dist("gloo", timeout_s=60)
    try:
        bench.barrier()
        slow = bench.reduce_max(1.0 + 2.0 * rank)      # rank 1 is the slowest: 3.0 s
        value = bench.job_value(6.0e12, slow, ws)      # 2 ranks x 6 TFLOP each over 3 s
        # the reference arm prints on rank 0 only; other ranks return without work
        args = bench.parse_args(["--impl", "reference", "--gpus", str(world), "--steps", "1", "--warmup", "0"])
        ran = None
        if rank != 0:
            ran = bench.run_reference(args)
        bench.barrier()
        out.put((rank, ws, r, slow, value, ran))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a gloo rank did not finish")
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ws, r, slow, value, ran in res:
        assert ws == 2 and r == rank
        assert slow == 3.0
        assert value == pytest.approx(4.0)             # 12 TFLOP / 3 s
        assert ran is None


def test_single_process_helpers_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(2.5) == 2.5
    bench.barrier()
    assert bench.job_value(1e12, 0.5, 1) == pytest.approx(2.0)

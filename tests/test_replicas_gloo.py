"""The multi-process replicas path of bench.py on CPU: two gloo ranks go through the same
process-group setup, barrier, max-over-ranks timing and whole-job rate as
`bench.py --gpus N` does with NCCL (the decode path itself has no collective)."""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(None, backend="gloo")
    bench.barrier(w)
    ms = 10.0 + 5.0 * r                                   # rank 1 is the slow one
    ms_max = bench.max_over_ranks(ms, w)
    out[r] = (w, ms_max, bench.whole_job_rate(w, 100, ms_max))
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_gloo_ranks_time_by_the_slowest_and_sum_the_work():
    world = 2
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r in range(world):
        w, ms_max, rate = res[r]
        assert w == world
        assert ms_max == 15.0                             # every rank sees the max
        assert abs(rate - world * 100 / 0.015) < 1e-6     # whole-job calls/s

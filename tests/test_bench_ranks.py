"""The multi-rank path of bench.py on CPU: world size 2 over gloo (no GPU).
The job's time is the slowest rank's and its tokens are all ranks'; the
reference arm runs on rank 0 only."""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r: step times 1 + r and 10 - r ms, 100 * (r + 1) tokens
        res = bench.aggregate_over_ranks(1.0 + rank, 10.0 - rank, 100 * (rank + 1), world, "cpu")
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_aggregate_over_two_gloo_ranks():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()  # no fork of a threaded process
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        assert out[r] == (2.0, 10.0, 300)  # max, max, sum on every rank


def test_single_rank_is_identity():
    assert bench.aggregate_over_ranks(1.5, 2.5, 7, 1, "cpu") == (1.5, 2.5, 7)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class Args:
        steps, warmup, gpus = 1, 3, 2

    assert bench.run_reference(Args, rank=1, world=2) == 0  # returns at once, prints nothing
    assert capsys.readouterr().out == ""

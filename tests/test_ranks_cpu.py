"""The multi-process side of bench.py on CPU: two gloo ranks (one process per
rank, as torchrun starts them) agree on the element-wise maximum of their
times, and the reference arm runs on rank 0 only."""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

torch = pytest.importorskip("torch")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_path):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank r reports times (r + 1, 10 - r, 3): the job's are the maxima
        got = bench.max_over_ranks(dist, [rank + 1.0, 10.0 - rank, 3.0], "cpu")

        class Args:
            steps, warmup, cpu_seconds, workload = 1, 0, 0.01, "dense_128x256x512"
        ref = bench.run_reference(Args, rank, world) if rank != 0 else "rank0"
        with open(out_path % rank, "w") as f:
            f.write(repr((got, ref)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rank_gating(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    out = str(tmp_path / "rank%d.txt")
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        got, ref = eval(open(out % rank).read())
        assert got == [2.0, 10.0, 3.0]
        if rank != 0:
            assert ref is None  # the reference arm prints on rank 0 only

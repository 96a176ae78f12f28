"""The bench's multi-GPU bookkeeping (replicas only: no data exchange) with two gloo ranks on
the CPU: the job time is the slowest rank's, and the whole-job figure divides by every
rank's layer-steps."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        dist.barrier()
        t = bench.max_over_ranks(10.0 * rank + 1.0, world, "cpu")  # per-rank times 1.0, 11.0
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(repr(t))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks(tmp_path):
    torch = pytest.importorskip("torch")
    import socket
    import torch.multiprocessing as mp
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    mp.start_processes(_rank, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    vals = [float((tmp_path / f"r{r}.txt").read_text()) for r in range(2)]
    assert vals == [11.0, 11.0]


def test_job_figure_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # 2 replicas, 10 steps of 8 layers in 1.0 ms: 160 layer-steps -> 6.25 us each
    assert bench.job_us_per_layer_step(1.0, 2, 10, 8) == pytest.approx(6.25)
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5

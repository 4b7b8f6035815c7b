"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (spawned processes)
take the barrier and the max over ranks of a time, draw independent replicas of the
workload, and the whole-job rate is the units of all ranks over the slowest rank's
time.  The path itself has no exchange between ranks (replicas only)."""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime
    import hashlib
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from gated_deltanet_sequence_delta_b200 import inputs as I
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ops = bench.RankOps(dist, torch.device("cpu"))
        ops.barrier()
        local_ms = 1.0 + 2.5 * rank          # rank 1 is the slow one
        ms_max = ops.max(local_ms)
        # each rank's replica of a small workload: different draws per rank
        inp = I.make_prefill(1, 128, 2, 2, 64, 64, io_dtype=I.BF16, seed=bench.replica_seed(2, rank))
        digest = hashlib.sha256(inp.q.data.tobytes()).hexdigest()
        rate = bench.whole_job_rate(world, 32768, ms_max)
        ops.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{ms_max} {rate} {digest}\n")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    rows = [open(tmp_path / f"rank{r}.txt").read().split() for r in range(world)]
    ms = [float(r[0]) for r in rows]
    rates = [float(r[1]) for r in rows]
    digests = [r[2] for r in rows]
    assert ms == [3.5, 3.5]                              # the max over ranks, seen by every rank
    assert rates[0] == rates[1] == pytest.approx(2 * 32768 / 3.5e-3)
    assert digests[0] != digests[1]                      # independent replicas


def test_single_process_ops_are_local():
    sys.path.insert(0, ROOT)
    import bench
    ops = bench.RankOps()
    ops.barrier()
    assert ops.max(1.25) == 1.25
    assert bench.replica_seed(2, 0) == 2
    assert bench.whole_job_rate(1, 1000, 1.0) == pytest.approx(1e6)

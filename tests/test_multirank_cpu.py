"""The N > 1 plumbing of bench.py on CPU: two gloo ranks (replicas only -- the path has no
exchange step).  Checks the max-over-ranks device time, the weak-scaling whole-job
throughput, and that only rank 0 runs and reports the reference (CPU oracle) arm."""
import argparse
import json
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


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(1.5 + rank, world, "cpu")
        args = argparse.Namespace(steps=1, warmup=0)
        line = bench.run_reference(args, rank, world)
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max_ms": t, "line": line}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert all(r["max_ms"] == 2.5 for r in res)        # the slowest rank's time on every rank
    assert res[1]["line"] is None                      # the reference arm runs on rank 0 only
    line = res[0]["line"]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_whole_job_throughput_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_gbs(1, 2.5e9, 1.0)
    assert one == pytest.approx(2500.0)
    assert bench.whole_job_gbs(4, 2.5e9, 1.0) == pytest.approx(4 * one)
    assert bench.whole_job_gbs(4, 2.5e9, 2.0) == pytest.approx(2 * one)

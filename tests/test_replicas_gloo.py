"""The multi-rank (replica) path of bench.py on CPU with the gloo backend,
world size 2: the slowest rank's time is what every rank reports, the
whole-job value counts every rank's work, and the reference arm runs on
rank 0 only."""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        # rank r "took" 10 * (r + 1) ms
        slowest = bench.max_over_ranks(torch, 10.0 * (rank + 1), world, torch.device("cpu"))
        value = bench.whole_job_tflops(1.0e12, world, slowest)

        class A:
            steps, warmup = 1, 0
        # non-zero ranks of the reference arm do no work and print nothing
        rc = bench.run_reference(A(), world, rank) if rank != 0 else 0
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"slowest": slowest, "value": value, "rc": rc}, f)
    finally:
        dist.destroy_process_group()


def test_replica_timing_and_value_over_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for r in res:
        assert r["slowest"] == pytest.approx(20.0)           # max over ranks, on every rank
        assert r["value"] == pytest.approx(1.0e12 * 2 / 20e-3 / 1e12)  # both ranks' flops / slowest time
    assert res[1]["rc"] == 0

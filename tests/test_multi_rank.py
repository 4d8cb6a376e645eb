"""The N > 1 path of bench.py on CPU: two gloo ranks exercise the barrier,
the max-over-ranks timing and the whole-job throughput that rank 0 reports,
and the reference arm's rule that only rank 0 runs it.  (The GPU pool gives
one GPU per call; the replicas share no data-path collective.)"""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

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
        ms = 10.0 * (rank + 1)  # rank 1 is the slower one
        bench.barrier(world)
        ms_max = bench.max_over_ranks(ms, world)
        value = bench.job_throughput(1000.0, ms_max, world)
        # the reference arm: every rank but 0 returns at once, printing nothing
        buf = io.StringIO()
        ref = None
        if rank != 0:
            class A:
                workload, policy, steps, warmup = "tiny_f32", "cumutil", 1, 0
            with redirect_stdout(buf):
                ref = bench.run_reference(A, world, rank)
        bench.barrier(world)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"ms_max": ms_max, "value": value, "ref_out": buf.getvalue(),
                       "ref_ret": ref}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_timing_and_job_value(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for r in res:
        assert r["ms_max"] == 20.0                     # the slowest rank's time on every rank
        assert r["value"] == pytest.approx(1e5)        # 2 ranks x 1000 units / 20 ms
    assert res[1]["ref_out"] == "" and res[1]["ref_ret"] is None

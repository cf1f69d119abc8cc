"""The multi-process plumbing of bench.py on the CPU: two gloo ranks.

One process per GPU runs independent replicas (no collective on the data
path); the only cross-rank steps are the barrier around the timed region and
the max over ranks of the measured times.  Here two CPU processes check that
every rank gets the slowest rank's time, that the whole-job rate counts both
replicas, and that only rank 0 of the reference arm prints its line.
"""
import io
import json
import os
import socket
import sys
import types
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(1.5 + rank, world, "cpu")   # rank 1 is the slower one
        rate = bench.job_throughput(world, 2.0e12, t)
        dist.barrier()
        buf = io.StringIO()
        args = types.SimpleNamespace(steps=1, warmup=0, gpus=world)
        with redirect_stdout(buf):
            bench.run_reference(args, rank, world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"t": t, "rate": rate, "stdout": buf.getvalue()}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_the_slowest_time_and_rank0_alone_reports(tmp_path):
    port = _free_port()
    mp.spawn(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    r0 = json.load(open(tmp_path / "rank0.json"))
    r1 = json.load(open(tmp_path / "rank1.json"))
    assert r0["t"] == r1["t"] == 2.5
    assert r0["rate"] == pytest.approx(2 * 2.0e12 / 2.5e-3 / 1e12)
    assert r1["stdout"] == ""
    line = json.loads(r0["stdout"].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"

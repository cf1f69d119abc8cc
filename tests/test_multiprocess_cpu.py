"""The multi-process plumbing of bench.py on the CPU: two gloo ranks.

One process per GPU, data parallel: each rank runs the layer on its own token
shard with the replicated NF4 weight and adapter, and the one exchange of a
step is the sum of dA and dB over ranks.  The other cross-rank steps are the
barrier around the timed region and the max over ranks of the measured times.
Here two CPU processes check that every rank gets the slowest rank's time,
that the whole-job rate counts both ranks, that only rank 0 of the reference
arm prints its line, and that the summed per-shard gradients (the oracle's,
on each half of the tiny workload's tokens) equal the full-batch gradients.
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


def _grad_worker(rank, world, port, out_dir):
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    from bit_nf4_quantized_quantize_b200 import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = synth.layer_inputs("tiny")
        f = lambda k: synth.bf16_bits_to_f32(inp[k]).astype(np.float64)
        codes, q8, s2, _ = oracle.quantize_nf4_dq(inp["W"].reshape(-1))
        _, wb = oracle.dequant(codes, q8, s2, inp["N"] * inp["K"])
        What = synth.bf16_bits_to_f32(wb).astype(np.float64).reshape(inp["N"], inp["K"])
        X, dY = f("X"), f("dY")
        shard = slice(rank * (inp["M"] // world), (rank + 1) * (inp["M"] // world))   # this rank's tokens
        _, dA, dB = oracle.linear_bwd(X[shard], What, f("A"), f("B"), dY[shard], inp["alpha"])
        tA, tB = torch.from_numpy(dA.copy()), torch.from_numpy(dB.copy())
        bench.sync_adapter_grads(tA, tB, world)
        if rank == 0:
            _, dA_full, dB_full = oracle.linear_bwd(X, What, f("A"), f("B"), dY, inp["alpha"])
            np.save(os.path.join(out_dir, "sum_dA.npy"), tA.numpy())
            np.save(os.path.join(out_dir, "sum_dB.npy"), tB.numpy())
            np.save(os.path.join(out_dir, "full_dA.npy"), dA_full)
            np.save(os.path.join(out_dir, "full_dB.npy"), dB_full)
    finally:
        dist.destroy_process_group()


def test_adapter_gradients_summed_over_token_shards_equal_the_full_batch(tmp_path):
    import numpy as np
    port = _free_port()
    mp.spawn(_grad_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    for g in ("dA", "dB"):
        got, ref = np.load(tmp_path / f"sum_{g}.npy"), np.load(tmp_path / f"full_{g}.npy")
        assert np.abs(ref).max() > 0
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-15 * np.abs(ref).max()), g

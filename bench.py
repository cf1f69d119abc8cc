#!/usr/bin/env python3
"""Benchmark of the QLoRA NF4 linear layer on B200.

Workload (one GPU): a single 4096 x 4096 frozen layer, NF4 + double quant,
M = 4096 tokens (4 x 1024), LoRA r = 64, alpha = 16, seeded synthetic inputs
(W ~ N(0, 0.02^2), X, dY ~ N(0, 1), A ~ N(0, 1/4096), B ~ N(0, 0.01^2)).
One step = the whole hot path once: quantize + double-quantize W, forward
(U = X A^T, Y = X dequant(W)^T + s U B^T), backward (V, dX, dA, dB).

Metric: algorithmic fwd+bwd FLOP of the step / device time of the step
(TFLOP/s); the quantize GB/s and per-kernel times are reported beside it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun, data parallel: one process per GPU, each with its
own tokens of the same shape (weak scaling) and a replica of the weight and
the adapter; the step ends with an NCCL all-reduce of dA and dB.  --impl
reference times the CPU oracle on the same workload (a bounded sample of it
per step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "train4096"
N_OUT, K_IN, M_TOK, RANK, ALPHA = 4096, 4096, 4096, 64, 16.0
METRIC = "QLoRA linear fwd+bwd TFLOP/s and quantize GB/s; % of roofline vs CPU oracle"
UNIT = "TFLOP/s"
L2_FLUSH_BYTES = 256 << 20
CPU_SAMPLE_TOKENS = 4096      # cpu_baseline: tokens of the oracle's sample step (the whole step)
REF_SAMPLE_TOKENS = 64        # --impl reference: tokens per sampled step


class L2Flush:
    """L2 flush between timed iterations: a write of L2_FLUSH_BYTES, then a
    read of a second buffer of the same size, so that the lines the write
    left dirty are written back here rather than inside the next timed
    kernel (which would otherwise pay for up to an L2's worth of write-back
    traffic that is not its own)."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.acc = torch.zeros((), dtype=torch.float32, device=dev)

    def __call__(self, i=0):
        import torch
        self.w.fill_(float(i))
        torch.sum(self.r, dim=0, out=self.acc)


def step_flops(M, N, K, r):
    """Algorithmic FLOP of fwd + bwd: main 4MNK, LoRA fwd 2Mr(K+N), LoRA bwd 2Mr(N+K) + 2rMK + 2NMr."""
    return 4 * M * N * K + 2 * M * r * (K + N) + 2 * M * r * (N + K) + 2 * r * M * K + 2 * N * M * r


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest x over all ranks (every rank gets it); x itself on one rank.  Times of a
    multi-GPU run are the slowest rank's."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sync_adapter_grads(dA, dB, world: int) -> None:
    """The data-parallel exchange of a step: every rank holds the gradients of its own token
    shard, and the adapter's gradients are their sum over ranks (the frozen NF4 weight and the
    adapter are replicated; dX stays with its shard).  One all-reduce each of dA and dB
    (r (N + K) fp32), on the stream the kernels ran on."""
    if world <= 1:
        return
    import torch.distributed as dist
    dist.all_reduce(dA, op=dist.ReduceOp.SUM)
    dist.all_reduce(dB, op=dist.ReduceOp.SUM)


def job_throughput(world: int, units_per_rank: float, ms: float, scale: float = 1e12) -> float:
    """Whole-job rate: the units all ranks processed (replicas: world x per rank) / the step time."""
    return world * units_per_rank / (ms * 1e-3) / scale


def quant_bytes(N, K):
    """Algorithmic quantize traffic: fp32 W in, packed codes + q8 + s2 out."""
    n = N * K
    nb = n // 64
    return 4 * n + n // 2 + nb + 4 * ((nb + 255) // 256)


def kernel_flops(kind, M, N, K, r):
    if kind == "fwd_fused":
        return 2 * M * N * K + 2 * M * N * r
    if kind == "dx_fused":
        return 2 * M * N * K + 2 * M * K * r
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sustained=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# Device sources of each timed kernel kind (csrc/): a capture's DRAM traffic
# stays valid while these files are unchanged.
KERNEL_SOURCES = {
    "fwd_fused": ("fused2_tc.cuh", "gemm_tc.cuh", "ptx_sm100.cuh"),
    "dx_fused": ("fused2_tc.cuh", "gemm_tc.cuh", "ptx_sm100.cuh"),
    "quantize": ("quantize.cuh", "ptx_sm100.cuh"),
    "lora_gemm": ("lora_tc.cuh", "ptx_sm100.cuh"),
    "grad_gemm": ("lora_tc.cuh", "ptx_sm100.cuh"),
}


def kernel_source_hash(kind):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_nf4_quantized_quantize_b200", "csrc")
    for f in KERNEL_SOURCES[kind]:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def load_traffic(kind):
    """Per-launch DRAM bytes of `kind` from the committed ncu summary, if it matches these sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(kind)
    if not e or kind not in KERNEL_SOURCES or e.get("source_hash") != kernel_source_hash(kind):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        busy = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


def make_inputs(M=M_TOK, N=N_OUT, K=K_IN, r=RANK, alpha=ALPHA):
    from bit_nf4_quantized_quantize_b200 import synth
    return synth.layer_inputs(WORKLOAD, M=M, shape=(N, K), r=r, alpha=alpha)


# ---------------------------------------------------------------------------- CPU oracle
def oracle_step(inp, M_s):
    """One sampled step on the CPU oracle: quantize the whole W, then fwd + bwd on M_s tokens."""
    import oracle
    from bit_nf4_quantized_quantize_b200 import synth
    N, K, alpha = inp["N"], inp["K"], inp["alpha"]
    t0 = time.perf_counter()
    codes, q8, s2, _ = oracle.quantize_nf4_dq(inp["W"].reshape(-1))
    t1 = time.perf_counter()
    _, wb = oracle.dequant(codes, q8, s2, N * K)
    What = synth.bf16_bits_to_f32(wb).astype(np.float64).reshape(N, K)
    f = lambda k: synth.bf16_bits_to_f32(inp[k]).astype(np.float64)
    X, A, B, dY = f("X")[:M_s], f("A"), f("B"), f("dY")[:M_s]
    t2 = time.perf_counter()
    oracle.linear_fwd(X, What, A, B, alpha)
    oracle.linear_bwd(X, What, A, B, dY, alpha)
    t3 = time.perf_counter()
    return dict(quant_s=t1 - t0, linear_s=t3 - t2, total_s=(t1 - t0) + (t3 - t2))


def cpu_baseline(inp):
    import oracle
    N, K, r = inp["N"], inp["K"], inp["r"]
    t = oracle_step(inp, CPU_SAMPLE_TOKENS)
    fl = step_flops(CPU_SAMPLE_TOKENS, N, K, r)
    return {"value": fl / t["linear_s"] / 1e12, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": (f"oracle fwd+bwd on {CPU_SAMPLE_TOKENS} of the {M_TOK} tokens (fp64, full N=K=4096, r=64) "
                       f"took {t['linear_s']:.2f} s; quantize+DQ of the full 4096x4096 W took {t['quant_s']:.2f} s "
                       f"= {quant_bytes(N, K) / t['quant_s'] / 1e9:.3f} GB/s"),
            "quantize_gbs": quant_bytes(N, K) / t["quant_s"] / 1e9}


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    inp = make_inputs()
    N, K, r = inp["N"], inp["K"], inp["r"]
    for _ in range(args.warmup):
        oracle_step(inp, REF_SAMPLE_TOKENS)
    times = [oracle_step(inp, REF_SAMPLE_TOKENS) for _ in range(args.steps)]
    lin = sum(t["linear_s"] for t in times) / len(times)
    qs = sum(t["quant_s"] for t in times) / len(times)
    fl = step_flops(REF_SAMPLE_TOKENS, N, K, r)
    value = fl / lin / 1e12
    sample = (f"each step: oracle quantize+DQ of the full 4096x4096 W ({qs:.2f} s) and fp64 fwd+bwd on "
              f"{REF_SAMPLE_TOKENS} of the {M_TOK} tokens ({lin:.2f} s); value = that sample's FLOP / its time")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": (lin + qs) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "train4096: one 4096x4096 NF4+DQ layer, M=4096 tokens, r=64, alpha=16; "
                                   "step = quantize + fwd + bwd (sampled tokens on the CPU)",
                       "N": N_OUT, "K": K_IN, "M": M_TOK, "r": RANK, "alpha": ALPHA},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "quantize_gbs": quant_bytes(N, K) / qs / 1e9}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------- decode shapes
DECODE_N = DECODE_K = 4096
DECODE_RANK = 8
DECODE_COPIES = 32          # rotated weight copies: 32 x 8.65 MB = 277 MB, more than L2
DECODE_REPLAYS = 20
DECODE_SINGLES = 12          # single launches timed one at a time
DECODE_SLEEP_CYCLES = 200000  # about 100 us of GPU sleep before each single launch's first event


def decode_weight_bytes(N, K):
    """Algorithmic bytes a decode forward must read: packed codes + q8 + s2."""
    n = N * K
    nb = n // 64
    return n // 2 + nb + 4 * ((nb + 255) // 256)


def run_decode(q, dev, peaks):
    """Forward of one 4096 x 4096 NF4+DQ layer (r = 8) at M in {1, 4, 16}: a
    CUDA graph of 32 layers, each on its own copy of the weight, replayed;
    time per layer from CUDA events around the replays.  Also the time of a
    single stream launch between its own event pair."""
    import torch
    from bit_nf4_quantized_quantize_b200 import synth
    N, K, r = DECODE_N, DECODE_K, DECODE_RANK
    inp = synth.layer_inputs("decode", M=16)
    W = torch.from_numpy(inp["W"]).to(dev)
    codes, q8, s2 = q.qlora_quantize_nf4_dq(W)
    copies = [(codes.clone(), q8.clone(), s2.clone()) for _ in range(DECODE_COPIES)]
    A = torch.from_numpy(inp["A"].view(np.int16)).view(torch.bfloat16).to(dev)
    B = torch.from_numpy(inp["B"].view(np.int16)).view(torch.bfloat16).to(dev)
    wbytes = decode_weight_bytes(N, K)
    out = {}
    for M in (1, 4, 16):
        X = torch.from_numpy(inp["X"][:M].view(np.int16)).view(torch.bfloat16).to(dev)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(q.qlora_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)

        def layers():
            for c in copies:
                q.qlora_linear_fwd(*c, N, K, X, A, B, inp["alpha"], Y=Y, workspace=ws)

        layers()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                layers()
        torch.cuda.synchronize()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(DECODE_REPLAYS):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (DECODE_REPLAYS * DECODE_COPIES)
        gbs = wbytes / (us * 1e-6) / 1e9
        # one launch alone (stream launch, no graph), each on a weight copy last read 31
        # launches earlier (so out of L2), between its own event pair; a GPU-side sleep in
        # front of the first event lets the host enqueue the launch before the GPU reaches it,
        # so the time is the GPU's and not the host's launch overhead
        single = []
        for i in range(DECODE_SINGLES):
            c = copies[i % DECODE_COPIES]
            torch.cuda._sleep(DECODE_SLEEP_CYCLES)
            e0.record()
            q.qlora_linear_fwd(*c, N, K, X, A, B, inp["alpha"], Y=Y, workspace=ws)
            e1.record()
            torch.cuda.synchronize()
            single.append(e0.elapsed_time(e1) * 1e3)
        single_us = float(np.median(single[2:]))
        out[str(M)] = {"us_per_layer": us, "gbs": gbs, "frac": gbs / peaks["hbm_gbs"],
                       "single_launch_us": single_us}
        del g
    rc = q.qlora_device_status()
    if rc != 0:
        raise RuntimeError(f"device status after the decode region: {q.qlora_strerror(rc)}")
    return {"workload": f"one {N}x{K} NF4+DQ layer, forward, r={r}, alpha=16; CUDA graph of {DECODE_COPIES} layers "
                        f"on rotated weight copies ({DECODE_COPIES * wbytes / 1e6:.0f} MB, more than L2)",
            "single_launch_timing": "median of single stream launches between their own event pair, each on a weight "
                                    "copy out of L2, enqueued behind a GPU sleep so that the host's launch time is "
                                    "hidden; the launch latency after a timing event is included",
            "bound": "hbm", "algorithmic_bytes_per_layer": wbytes, "peak_gbs": peaks["hbm_gbs"],
            "unit": "GB/s", "by_tokens": out}


# ---------------------------------------------------------------------------- larger configurations
STACK_7B = [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]   # q, k, v, o, gate, up, down
LINEARS_65B = [(8192, 8192), (22016, 8192)]
STREAM_CHUNKS, STREAM_CHUNK_PARAMS = 30, 1 << 26   # 30 x 256 MiB of fp32 = 2.01e9 parameters


def gpu_weight(gen, N, K, kind, dev):
    """Seeded synthetic weight on the GPU: N(0, 0.02^2), optionally with 0.1% +-6 sigma outliers, or
    Student-t (4 degrees of freedom) scaled to std 0.02."""
    import torch
    if kind == "student_t4":
        z = torch.randn(N, K, generator=gen, device=dev)
        chi2 = sum(torch.randn(N, K, generator=gen, device=dev) ** 2 for _ in range(4))
        return z / torch.sqrt(chi2 / 4) * (0.02 / 2 ** 0.5)
    w = torch.randn(N, K, generator=gen, device=dev) * 0.02
    if kind == "normal+outliers":
        mask = torch.rand(N, K, generator=gen, device=dev) < 1e-3
        sign = torch.where(torch.rand(N, K, generator=gen, device=dev) < 0.5, -1.0, 1.0)
        w = torch.where(mask, 0.12 * sign, w)
    return w


def time_region(fn, warmup, reps):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


QUANT_BURST_COPIES, QUANT_BURST_REPS = 8, 5


def run_quantize_burst(q, dev, W, peaks):
    """The step's quantizer launched back to back over QUANT_BURST_COPIES copies of the
    4096 x 4096 weight (537 MB, more than L2), as a stream of layers would be quantized:
    device time per launch from one event pair around each burst."""
    import torch
    N, K = W.shape
    copies = [W.clone() for _ in range(QUANT_BURST_COPIES)]
    codes = torch.empty(N * K // 2, dtype=torch.uint8, device=dev)
    q8 = torch.empty(N * K // 64, dtype=torch.uint8, device=dev)
    s2 = torch.empty((N * K // 64 + 255) // 256, dtype=torch.float32, device=dev)

    def burst():
        for c in copies:
            q.qlora_quantize_nf4_dq(c, codes, q8, s2)

    ms = time_region(burst, 2, QUANT_BURST_REPS) / QUANT_BURST_COPIES
    gbs = quant_bytes(N, K) / (ms * 1e-3) / 1e9
    del copies
    return {"ms_per_launch": ms, "gbs": gbs, "frac": gbs / peaks["hbm_gbs"],
            "how": f"{QUANT_BURST_COPIES} launches back to back on distinct weight copies "
                   f"({QUANT_BURST_COPIES * 4 * N * K / 1e6:.0f} MB of fp32 input), {QUANT_BURST_REPS} bursts"}


def run_linear_stack(q, dev, shapes, M, r, alpha, kind, seed, peaks, warmup=2, reps=5):
    """fwd through every linear, then bwd in reverse order; weights quantized once beforehand."""
    import torch
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    layers = []
    for (N, K) in shapes:
        W = gpu_weight(gen, N, K, kind, dev)
        codes, q8, s2 = q.qlora_quantize_nf4_dq(W)
        del W
        L = dict(N=N, K=K, codes=codes, q8=q8, s2=s2,
                 X=torch.randn(M, K, generator=gen, device=dev).bfloat16(),
                 A=(torch.randn(r, K, generator=gen, device=dev) / K ** 0.5).bfloat16(),
                 B=(torch.randn(N, r, generator=gen, device=dev) * 0.01).bfloat16(),
                 dY=torch.randn(M, N, generator=gen, device=dev).bfloat16(),
                 Y=torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                 U=torch.empty(M, r, dtype=torch.bfloat16, device=dev),
                 dX=torch.empty(M, K, dtype=torch.bfloat16, device=dev),
                 dA=torch.empty(r, K, dtype=torch.float32, device=dev),
                 dB=torch.empty(N, r, dtype=torch.float32, device=dev),
                 ws=torch.empty(q.qlora_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev))
        layers.append(L)

    def step():
        for L in layers:
            q.qlora_linear_fwd(L["codes"], L["q8"], L["s2"], L["N"], L["K"], L["X"], L["A"], L["B"], alpha,
                               Y=L["Y"], U_save=L["U"], workspace=L["ws"])
        for L in reversed(layers):
            q.qlora_linear_bwd(L["codes"], L["q8"], L["s2"], L["N"], L["K"], L["X"], L["A"], L["B"], alpha,
                               L["dY"], U_saved=L["U"], dX=L["dX"], dA=L["dA"], dB=L["dB"], workspace=L["ws"])

    ms = time_region(step, warmup, reps)
    rc = q.qlora_device_status()
    if rc != 0:
        raise RuntimeError(f"device status after the linear stack: {q.qlora_strerror(rc)}")
    fl = sum(step_flops(M, N, K, r) for (N, K) in shapes)
    tf = fl / (ms * 1e-3) / 1e12
    return {"shapes": [f"{N}x{K}" for (N, K) in shapes], "M": M, "r": r, "ms_per_step": ms,
            "algorithmic_flop": fl, "tflops": tf, "frac_of_bf16_peak": tf / peaks["bf16"],
            "steps": reps, "warmup": warmup}


def run_quantize_stream(q, dev, peaks, seed=5, reps=3):
    """NF4 + DQ over 30 chunks of 2^26 Student-t parameters (256 MiB of fp32 each), one launch per chunk."""
    import torch
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    n = STREAM_CHUNK_PARAMS
    W = torch.empty(STREAM_CHUNKS, n, dtype=torch.float32, device=dev)
    for c in range(STREAM_CHUNKS):
        W[c] = gpu_weight(gen, 1, n, "student_t4", dev).view(-1)
    nc, nb, ng = q._binding.quant_sizes(n // 4096, 4096)
    codes = torch.empty(STREAM_CHUNKS, nc, dtype=torch.uint8, device=dev)
    q8 = torch.empty(STREAM_CHUNKS, nb, dtype=torch.uint8, device=dev)
    s2 = torch.empty(STREAM_CHUNKS, ng, dtype=torch.float32, device=dev)

    def one_pass():
        for c in range(STREAM_CHUNKS):
            q.qlora_quantize_nf4_dq(W[c].view(n // 4096, 4096), codes[c], q8[c], s2[c])

    ms = time_region(one_pass, 1, reps)
    rc = q.qlora_device_status()
    if rc != 0:
        raise RuntimeError(f"device status after the quantize stream: {q.qlora_strerror(rc)}")
    byts = STREAM_CHUNKS * quant_bytes(n // 4096, 4096)
    gbs = byts / (ms * 1e-3) / 1e9
    return {"params": STREAM_CHUNKS * n, "chunks": STREAM_CHUNKS, "chunk_bytes_fp32": 4 * n, "ms_per_pass": ms,
            "algorithmic_bytes": byts, "gbs": gbs, "frac": gbs / peaks["hbm_gbs"], "passes": reps}


def run_quant_variant(q, dev, peaks, variant, reps=20):
    """The train4096 layer with another form of the second quantization stage
    ("single": off, 4 B read and 0.5 + 4/64 B written per weight; "fp8": the
    FP8-E4M3 reading, the same bytes as the linear form): quantize GB/s and
    fwd+bwd TFLOP/s."""
    import torch
    N, K, M, r, alpha = N_OUT, K_IN, M_TOK, RANK, ALPHA
    gen = torch.Generator(device=dev)
    gen.manual_seed(3)
    W = gpu_weight(gen, N, K, "normal", dev)
    codes = torch.empty(N * K // 2, dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    if variant == "single":
        q8 = None
        s2 = torch.empty(N * K // 64, dtype=torch.float32, device=dev)
        qbytes = 4 * N * K + N * K // 2 + 4 * (N * K // 64)
        qfn = lambda: q.qlora_quantize_nf4(W, codes, s2)
    else:
        q8 = torch.empty(N * K // 64, dtype=torch.uint8, device=dev)
        s2 = torch.empty((N * K // 64 + 255) // 256, dtype=torch.float32, device=dev)
        qbytes = quant_bytes(N, K)
        qfn = lambda: q.qlora_quantize_nf4_dq_fp8(W, codes, q8, s2)

    def quant():
        flush(0.0)
        qfn()

    # time the quantize launches alone: events around each, after an L2 flush
    for _ in range(3):
        quant()
    ev = []
    for _ in range(reps):
        flush(0.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        qfn()
        e1.record()
        ev.append((e0, e1))
    torch.cuda.synchronize()
    q_ms = sum(a.elapsed_time(b) for a, b in ev) / reps
    L = dict(X=torch.randn(M, K, generator=gen, device=dev).bfloat16(),
             A=(torch.randn(r, K, generator=gen, device=dev) / K ** 0.5).bfloat16(),
             B=(torch.randn(N, r, generator=gen, device=dev) * 0.01).bfloat16(),
             dY=torch.randn(M, N, generator=gen, device=dev).bfloat16())
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    U = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dA = torch.empty(r, K, dtype=torch.float32, device=dev)
    dB = torch.empty(N, r, dtype=torch.float32, device=dev)
    ws = torch.empty(q.qlora_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)

    def step():
        q.qlora_linear_fwd(codes, q8, s2, N, K, L["X"], L["A"], L["B"], alpha, Y=Y, U_save=U, workspace=ws)
        q.qlora_linear_bwd(codes, q8, s2, N, K, L["X"], L["A"], L["B"], alpha, L["dY"], U_saved=U, dX=dX,
                           dA=dA, dB=dB, workspace=ws)

    ms = time_region(step, 3, 10)
    rc = q.qlora_device_status()
    if rc != 0:
        raise RuntimeError(f"device status after the {variant} quantization region: {q.qlora_strerror(rc)}")
    tf = step_flops(M, N, K, r) / (ms * 1e-3) / 1e12
    gbs = qbytes / (q_ms * 1e-3) / 1e9
    what = "second quantization stage off (4.5 bit/param)" if variant == "single" else \
        "FP8-E4M3 second quantization stage (4.127 bit/param)"
    return {"workload": f"train4096 layer, {what}",
            "quantize_gbs": gbs, "quantize_frac": gbs / peaks["hbm_gbs"], "quantize_algorithmic_bytes": qbytes,
            "fwd_bwd_tflops": tf, "fwd_bwd_ms": ms}


def run_merge(q, dev, peaks, reps=10):
    """Adapter merge into the bf16 base of the train4096 layer (r = 64), then NF4 + DQ of the
    merged weight: time of each launch; the merge is fp64-issue bound (2 r fp64 ops per weight)."""
    import torch
    N, K, r, alpha = N_OUT, K_IN, RANK, ALPHA
    gen = torch.Generator(device=dev)
    gen.manual_seed(6)
    W = gpu_weight(gen, N, K, "normal", dev)
    A = (torch.randn(r, K, generator=gen, device=dev) / K ** 0.5).bfloat16()
    B = (torch.randn(N, r, generator=gen, device=dev) * 0.01).bfloat16()
    merged = torch.empty(N, K, dtype=torch.float32, device=dev)
    codes = torch.empty(N * K // 2, dtype=torch.uint8, device=dev)
    q8 = torch.empty(N * K // 64, dtype=torch.uint8, device=dev)
    s2 = torch.empty((N * K // 64 + 255) // 256, dtype=torch.float32, device=dev)
    m_ms = time_region(lambda: q.qlora_merge_adapter(W, A, B, alpha, out=merged), 2, reps)
    q_ms = time_region(lambda: q.qlora_quantize_nf4_dq(merged, codes, q8, s2), 2, reps)
    rc = q.qlora_device_status()
    if rc != 0:
        raise RuntimeError(f"device status after the merge region: {q.qlora_strerror(rc)}")
    fp64_ops = 2 * N * K * r
    return {"workload": "train4096 layer, r=64: merge into the bf16 base, then NF4+DQ of the merged weight",
            "merge_ms": m_ms, "merge_fp64_ops": fp64_ops, "merge_fp64_gops_per_s": fp64_ops / (m_ms * 1e-3) / 1e9,
            "requantize_ms": q_ms, "requantize_gbs": quant_bytes(N, K) / (q_ms * 1e-3) / 1e9}


def run_dropout(q, dev, peaks, p=0.05, reps=10):
    """The train4096 step's fwd+bwd with LoRA dropout p on the adapter input (the mask, a
    masked adapter term of dX and the masked dA come on top of the plain step's work)."""
    import torch
    N, K, M, r, alpha = N_OUT, K_IN, M_TOK, RANK, ALPHA
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)
    codes, q8, s2 = q.qlora_quantize_nf4_dq(gpu_weight(gen, N, K, "normal", dev))
    X = torch.randn(M, K, generator=gen, device=dev).bfloat16()
    A = (torch.randn(r, K, generator=gen, device=dev) / K ** 0.5).bfloat16()
    B = (torch.randn(N, r, generator=gen, device=dev) * 0.01).bfloat16()
    dY = torch.randn(M, N, generator=gen, device=dev).bfloat16()
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    U = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dA = torch.empty(r, K, dtype=torch.float32, device=dev)
    dB = torch.empty(N, r, dtype=torch.float32, device=dev)
    ws = torch.empty(q.qlora_workspace_bytes_dropout(M, N, K, r), dtype=torch.uint8, device=dev)
    # the state a training framework keeps for dropout's backward: the masked input and the mask
    Xd = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    keep = torch.empty(M * K // 32, dtype=torch.int32, device=dev)
    it = [0]

    def step():
        it[0] += 1   # a fresh mask every step: offset = step index
        q.qlora_linear_fwd_dropout(codes, q8, s2, N, K, X, A, B, alpha, p, 1234, it[0], Y=Y, U_save=U, Xd_save=Xd,
                                   keep_save=keep, workspace=ws)
        q.qlora_linear_bwd_dropout(codes, q8, s2, N, K, X, A, B, alpha, p, 1234, it[0], dY, U_saved=U, dX=dX, dA=dA,
                                   dB=dB, Xd_saved=Xd, keep_saved=keep, workspace=ws)

    ms = time_region(step, 3, reps)
    rc = q.qlora_device_status()
    if rc != 0:
        raise RuntimeError(f"device status after the dropout region: {q.qlora_strerror(rc)}")
    return {"workload": f"train4096 layer fwd+bwd with LoRA dropout p={p} on the adapter input; the forward "
                        "keeps the masked input and the keep bits for the backward",
            "fwd_bwd_ms": ms, "fwd_bwd_tflops": step_flops(M, N, K, r) / (ms * 1e-3) / 1e12}


def run_configs(q, dev, peaks):
    import torch
    out = {"data": "seeded synthetic, generated on the GPU (torch generator) with the distributions named "
                   "per config; weights quantized once, outside the timed region"}
    out["llama7b_stack"] = run_linear_stack(q, dev, STACK_7B, 2048, 64, 16.0, "normal+outliers", 4, peaks)
    torch.cuda.empty_cache()
    out["llama65b_linears"] = run_linear_stack(q, dev, LINEARS_65B, 8192, 64, 16.0, "student_t4", 5, peaks)
    torch.cuda.empty_cache()
    out["llama65b_quantize_stream"] = run_quantize_stream(q, dev, peaks)
    torch.cuda.empty_cache()
    out["train4096_single_quant"] = run_quant_variant(q, dev, peaks, "single")
    torch.cuda.empty_cache()
    out["train4096_fp8_dq"] = run_quant_variant(q, dev, peaks, "fp8")
    torch.cuda.empty_cache()
    out["train4096_merge_requantize"] = run_merge(q, dev, peaks)
    torch.cuda.empty_cache()
    out["train4096_dropout"] = run_dropout(q, dev, peaks)
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------- GPU
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import bit_nf4_quantized_quantize_b200 as q

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    q.load()
    inp = make_inputs()
    N, K, M, r, alpha = inp["N"], inp["K"], inp["M"], inp["r"], inp["alpha"]

    def pinned(a, dtype=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if dtype is not None:
            t = t.view(dtype)
        return t.pin_memory()

    hW = pinned(inp["W"])
    hX, hA, hB, hdY = (pinned(inp[k].view(np.int16), torch.bfloat16) for k in ("X", "A", "B", "dY"))
    W, X, A, B, dY = (t.to(dev) for t in (hW, hX, hA, hB, hdY))
    nc, nb, ng = q._binding.quant_sizes(N, K)
    codes = torch.empty(nc, dtype=torch.uint8, device=dev)
    q8 = torch.empty(nb, dtype=torch.uint8, device=dev)
    s2 = torch.empty(ng, dtype=torch.float32, device=dev)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    U = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dA = torch.empty(r, K, dtype=torch.float32, device=dev)
    dB = torch.empty(N, r, dtype=torch.float32, device=dev)
    ws = torch.empty(q.qlora_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)

    def step(Wd=W, Xd=X, dYd=dY, Ad=A, Bd=B):
        q.qlora_quantize_nf4_dq(Wd, codes, q8, s2)
        q.qlora_linear_fwd(codes, q8, s2, N, K, Xd, Ad, Bd, alpha, Y=Y, U_save=U, workspace=ws)
        q.qlora_linear_bwd(codes, q8, s2, N, K, Xd, Ad, Bd, alpha, dYd, U_saved=U, dX=dX, dA=dA, dB=dB,
                           workspace=ws)
        sync_adapter_grads(dA, dB, world)   # N > 1: sum the adapter gradients over the token shards

    def barrier():
        if world > 1:
            dist.barrier()

    if args.profile:
        # profiling case for ncu: one step to load the modules, one step to
        # capture, then decode forwards (r = 8) on the same weight: two at
        # M = 1, then two at M = 16.  Launches: [L2 flush write + L2 flush read
        # + 6 step kernels] x 2, then [adapter kernel + table kernel] x 2 (M = 1)
        # and 2 tensor-memory decode kernels (M = 16).
        from bit_nf4_quantized_quantize_b200 import synth
        dinp = synth.layer_inputs("decode", M=16)
        decA, decB = (torch.from_numpy(dinp[k].view(np.int16)).view(torch.bfloat16).to(dev) for k in ("A", "B"))
        for i in range(2):
            flush(float(i))
            step()
        for dm in (1, 1, 16, 16):
            decX = torch.from_numpy(dinp["X"][:dm].view(np.int16)).view(torch.bfloat16).to(dev)
            decY = torch.empty(dm, N, dtype=torch.bfloat16, device=dev)
            dws = torch.empty(q.qlora_workspace_bytes(dm, N, K, DECODE_RANK), dtype=torch.uint8, device=dev)
            q.qlora_linear_fwd(codes, q8, s2, N, K, decX, decA, decB, dinp["alpha"], Y=decY, workspace=dws)
        torch.cuda.synchronize()
        rc = q.qlora_device_status()
        print(json.dumps({"profile_case": WORKLOAD + " step + decode M=1, M=16", "device_status": rc}), flush=True)
        if rc != 0:
            raise RuntimeError(q.qlora_strerror(rc))
        return

    for i in range(args.warmup):
        flush(float(i))
        step()
    torch.cuda.synchronize()
    rc = q.qlora_device_status()
    if rc != 0:
        raise RuntimeError(f"device status after warm-up: {q.qlora_strerror(rc)}")

    # ---------------------------------------------------------------- timed region
    # Step events only: the library's kernels keep their programmatic-launch
    # overlap.  gpu_launches counts the library's launches inside the region.
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    n0 = q.qlora_launch_count()
    t_wall = time.perf_counter()
    for i in range(args.steps):
        flush(float(i))          # L2 flush between steps, outside the step's events
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    wall = time.perf_counter() - t_wall
    launches = q.qlora_launch_count() - n0
    barrier()
    clocks = sampler.stop()
    rc = q.qlora_device_status()
    if rc != 0:
        raise RuntimeError(f"device status after the timed region: {q.qlora_strerror(rc)}")
    step_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / args.steps, world, dev)

    # ---------------------------------------------------------------- per-kernel breakdown
    # The same steps again with a CUDA event pair around every library launch
    # (on the launching stream); these events serialise the launches, so the
    # per-kernel times are each kernel on its own.
    barrier()
    torch.cuda.synchronize()
    q.qlora_timing_enable(True)
    for i in range(args.steps):
        flush(float(i))
        step()
    torch.cuda.synchronize()
    kern = q.qlora_timing_collect()
    q.qlora_timing_enable(False)
    rc = q.qlora_device_status()
    if rc != 0:
        raise RuntimeError(f"device status after the breakdown region: {q.qlora_strerror(rc)}")

    # ---------------------------------------------------------------- end to end (host buffers)
    n_e2e = max(3, min(args.steps, 10))
    hY = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    hdX = torch.empty(M, K, dtype=torch.bfloat16).pin_memory()
    hdA = torch.empty(r, K, dtype=torch.float32).pin_memory()
    hdB = torch.empty(N, r, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hW, hX, hA, hB, hdY))
    d2h = sum(t.numel() * t.element_size() for t in (hY, hdX, hdA, hdB))
    e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_e2e)]
    # Uploads and downloads run on their own streams so that the two copy
    # directions overlap each other and the kernels: W goes up first (the
    # quantizer needs only W), then X, A, B (the forward), then dY (the
    # backward); Y comes down while dY goes up and the backward runs, then
    # dX, dA, dB.  The library calls stay on the current stream.
    cur = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    barrier()
    torch.cuda.synchronize()
    for i in range(n_e2e):
        flush(float(i))
        e_ev[i][0].record(cur)
        up.wait_stream(cur)
        with torch.cuda.stream(up):
            W.copy_(hW, non_blocking=True)
            w_up = up.record_event()
            X.copy_(hX, non_blocking=True)
            A.copy_(hA, non_blocking=True)
            B.copy_(hB, non_blocking=True)
            x_up = up.record_event()
            dY.copy_(hdY, non_blocking=True)
            dy_up = up.record_event()
        cur.wait_event(w_up)
        q.qlora_quantize_nf4_dq(W, codes, q8, s2)
        cur.wait_event(x_up)
        q.qlora_linear_fwd(codes, q8, s2, N, K, X, A, B, alpha, Y=Y, U_save=U, workspace=ws)
        down.wait_stream(cur)
        with torch.cuda.stream(down):
            hY.copy_(Y, non_blocking=True)
        cur.wait_event(dy_up)
        q.qlora_linear_bwd(codes, q8, s2, N, K, X, A, B, alpha, dY, U_saved=U, dX=dX, dA=dA, dB=dB,
                           workspace=ws)
        sync_adapter_grads(dA, dB, world)
        down.wait_stream(cur)
        with torch.cuda.stream(down):
            hdX.copy_(dX, non_blocking=True)
            hdA.copy_(dA, non_blocking=True)
            hdB.copy_(dB, non_blocking=True)
        cur.wait_stream(down)
        e_ev[i][1].record(cur)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in e_ev) / n_e2e, world, dev)
    # the copies must have carried the step's own results
    if not (torch.equal(hY, Y.cpu()) and torch.equal(hdX, dX.cpu()) and torch.equal(hdA, dA.cpu())
            and torch.equal(hdB, dB.cpu())):
        raise RuntimeError("end-to-end results differ from the device-resident step's")

    if rank != 0:
        return
    fl = step_flops(M, N, K, r)
    value = job_throughput(world, fl, step_ms)
    peaks = load_peaks()
    per_step = {k: {"ms_per_step": v[0] / args.steps, "launches_per_step": v[1] / args.steps,
                    "ms_per_launch": v[0] / v[1]} for k, v in kern.items()}
    dom = max(kern, key=lambda k: kern[k][0])
    dom_ms = kern[dom][0] / kern[dom][1]
    kf = kernel_flops(dom, M, N, K, r)
    long_region = wall > 1.0   # the breakdown region has the same length
    if kf is not None:
        peak = peaks["bf16_sustained"] if long_region else peaks["bf16"]
        achieved = kf / (dom_ms * 1e-3) / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": load_traffic(dom),
                "peak_source": f"{peaks['source']} bf16 dense "
                               f"{'sustained' if long_region else 'burst'} (timed region {wall:.2f} s)",
                "timing": "per-launch CUDA events on the launching stream, breakdown region of the same steps",
                "algorithmic_flop_per_launch": kf, "ms_per_launch": dom_ms}
    else:
        roof = {"kernel": dom, "bound": "hbm", "achieved": None, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": None, "traffic": load_traffic(dom)}
    qk = kern.get("quantize")
    quant_gbs = quant_bytes(N, K) / (qk[0] / qk[1] * 1e-3) / 1e9 if qk else None
    qburst = run_quantize_burst(q, dev, W, peaks)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "train4096: one 4096x4096 NF4+DQ layer, M=4096 tokens (4x1024), r=64, alpha=16; "
                               "step = quantize + fwd + bwd",
                   "N": N, "K": K, "M": M, "r": r, "alpha": alpha,
                   "l2": f"flushed between steps ({L2_FLUSH_BYTES >> 20} MiB write, then a {L2_FLUSH_BYTES >> 20} MiB read "
                         "that writes back the dirty lines; outside the step events)",
                   "parallelism": (f"data parallel x{world}: token shards, replicated NF4 weight and adapter, "
                                   "dA and dB summed over ranks (NCCL all-reduce) every step")
                                  if world > 1 else "1 GPU"},
        "roofline": roof,
        "quantize": {"gbs": qburst["gbs"], "peak_gbs": peaks["hbm_gbs"], "frac": qburst["frac"],
                     "ms_per_launch": qburst["ms_per_launch"], "timing": qburst["how"],
                     "single_launch_gbs": quant_gbs,
                     "single_launch_timing": "event pair around the step's one launch (breakdown region); "
                                             "includes the launch and event gaps",
                     "algorithmic_bytes": quant_bytes(N, K), "traffic": load_traffic("quantize")},
        "kernels": per_step,
        "gpu_launches": launches,
        "e2e": {"value": job_throughput(world, fl, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "copies": "pinned host buffers; uploads and downloads on two copy streams, overlapped with "
                          "each other and the kernels (W, then X/A/B, then dY up; Y down after the forward, "
                          "dX/dA/dB after the backward)"},
        "clocks": clocks,
    }
    line["decode"] = run_decode(q, dev, peaks)
    if not args.no_configs:
        line["configs"] = run_configs(q, dev, peaks)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inp)
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the 7B-stack / 65B-linear / quantize-stream measurements")
    ap.add_argument("--profile", action="store_true",
                    help="run two steps and exit (the case ncu captures); no timing")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the SALR linear layer Y = X (M.W)^T + (X A_cat) B_cat on B200.

One step is one salr_linear call.  The headline line is the largest single-GPU workload
of the configurations: W 28672 x 8192 bf16 (heavy-tailed), 50% per-row magnitude pruned
and bitmap-encoded, adapters 64 + 32 stacked to R = 96, X 8192 x 8192.
--workload/--tokens time another point of salr_synth.WORKLOADS as the headline instead.
Every configuration point (tiny 16; q_proj 1, 16; up_proj 2048; down_proj 1, 128, 4096;
large 16, 8192) is also timed the same way and reported under "per_config".  Prints one
JSON line (see --help).

Timing: W warm-up steps, then K steps queued back to back behind a short GPU sleep (so
that host launch overhead leaves no gaps), with CUDA events on the launching stream at the
two ends of the region; consecutive calls may overlap (programmatic dependent launch), as
consecutive layers would.  A second pass puts an event pair around every call and reports
their percentiles.  The weight/adapter set rotates over enough copies that the working set
exceeds twice the L2 (no step finds its weights in L2).

--impl reference times the fp64 CPU oracle on a bounded sample of the same workload
instead (each step: up to 64 tokens against up to 1024 output rows, on the host cores;
tokens/s counts full-layer tokens).  Under torchrun every rank runs an independent
replica (the layer has no data-path exchange); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import salr_synth as synth  # noqa: E402

METRIC = "SALR linear tokens/s + achieved fraction of HBM/tensor roofline on 1 B200"
WORKLOAD = "large"
M_TOKENS = 8192
SPARSITY = None  # None: the workload's own (0.5)
L2_BYTES = 126 * 1024 * 1024
# the headers each layer kernel is compiled from: a recorded DRAM-traffic figure stays
# valid while these are unchanged
KERNEL_SOURCES = {
    "salr_stream_kernel": ["sm100.cuh", "salr_block.cuh", "salr_decode.cuh", "salr_codec.cuh",
                           "salr_stream.cuh"],
    "salr_prefill_kernel": ["sm100.cuh", "salr_block.cuh", "salr_decode.cuh", "salr_codec.cuh",
                            "salr_stream.cuh", "salr_prefill.cuh"],
}


def workload():
    wl = synth.WORKLOADS[WORKLOAD]
    if SPARSITY is None:
        return wl
    # the library takes sparsity as a float32: use that value everywhere
    return dataclasses.replace(wl, sparsity=float(np.float32(SPARSITY)))


def algorithmic_bytes(N, K, R, M, keep):
    """Bytes the layer must move: bitmap, kept values, offset table, adapters (once),
    activations in and outputs out (padding and L2 re-reads excluded)."""
    return (N * K / 8 + 2 * N * keep + (N // 128) * (K // 64) * 4 + 2 * R * (K + N)
            + 2 * M * K + 2 * M * N)


def algorithmic_flops(N, K, R, M):
    return 2 * M * N * K + 2 * M * K * R + 2 * M * R * N


def kernel_hash(kname):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kname.split("<")[0]]:
        with open(os.path.join(ROOT, "sparse_rank_linear_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def max_over_ranks(value, ws, device):
    """The largest of every rank's value (a replica run ends when its slowest rank does);
    the value itself with one rank.  ``device`` is where the process group's backend
    keeps tensors: "cuda" for NCCL, "cpu" for gloo."""
    if ws <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(ws, steps, tokens, total_ms):
    """Tokens per second of the whole job: every rank processed ``steps`` calls of
    ``tokens`` tokens, and the job took the slowest rank's ``total_ms``."""
    return ws * steps * tokens / (total_ms * 1e-3)


def dense_lora_context(w_bits, x_bits, a_cat, b_cat, wl, M, steps, salr_total_ms):
    """Time the unpruned layer, Y = X W^T + (X A_cat) B_cat, with dense bf16 W through
    torch (cuBLAS), back to back over enough dense copies to exceed twice the L2.  Context
    for the pages' speedup-over-dense-LoRA claim; not part of the library."""
    import torch

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
            torch.bfloat16).cuda()

    N, K = wl.N, wl.K
    copies = max(1, min(16, int(np.ceil(2 * L2_BYTES / (2 * N * K)))))
    Ws = [dev(w_bits) for _ in range(copies)]
    A, B, X = dev(a_cat), dev(b_cat), dev(x_bits)

    def step(i):
        return torch.addmm((X @ A) @ B, X, Ws[i % copies].t())

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(int(2e9 * 40e-6 * steps) + 10_000_000)
    e0.record()
    for i in range(steps):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    del Ws
    return {"ms_per_step": ms / steps, "tokens_per_s": steps * M / (ms * 1e-3),
            "salr_speedup": ms / salr_total_ms, "dense_copies": copies,
            "note": "torch bf16 (cuBLAS) X W^T + (X A_cat) B_cat with the unpruned W, "
                    "same GPU and steps; context only"}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return ws, int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0"))


def max_sm_mhz():
    try:
        out = subprocess.run(["nvidia-smi", "--id=0", "--query-gpu=clocks.max.sm",
                              "--format=csv,noheader,nounits"], capture_output=True, text=True,
                             timeout=20).stdout
        return float(out.strip().splitlines()[0])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        rows = []
        for line in open(self.path):
            p = [v.strip() for v in line.split(",")]
            if len(p) >= 9:
                rows.append(p)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def oracle_sample_fn(wl, M, rows):
    """The fp64 oracle on a bounded sample of one step: ``M`` tokens against the first
    ``rows`` output rows of W (mask, pruned weight and adapters' columns prepared
    untimed).  The work per (token, output row) is that of the full layer."""
    import oracle
    w = synth.weight(wl, rows=np.arange(rows))
    wp = oracle.prune(w, oracle.magnitude_mask(w, wl.sparsity))
    x = synth.activations(wl, M)
    ad = [(a, b[:, :rows]) for a, b in synth.adapters(wl)]
    return lambda: oracle.linear(x, wp, ad)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


# bounded oracle sample: at most this many tokens and output rows per step
ORACLE_TOKENS = 64
ORACLE_ROWS = 1024


def oracle_sample(wl, M):
    """(tokens, rows) of one oracle step and the factor that turns its tokens into
    full-layer tokens (a sampled step covers rows / N of each token's outputs)."""
    mo, ro = min(M, ORACLE_TOKENS), min(wl.N, ORACLE_ROWS)
    return mo, ro, ro / wl.N


def time_oracle(wl, M, steps=None, budget_s=10.0):
    """Oracle steps in a bounded time (or a fixed count); returns (steps, seconds,
    full-layer tokens per second, sample description)."""
    mo, ro, frac = oracle_sample(wl, M)
    step = oracle_sample_fn(wl, mo, ro)
    step()  # warm
    t0 = time.perf_counter()
    n = 0
    while True:
        step()
        n += 1
        el = time.perf_counter() - t0
        if (steps is not None and n >= steps) or (steps is None and el >= budget_s):
            break
    sample = (f"{n} steps of {mo} of the {M} tokens x {ro} of the {wl.N} output rows "
              f"({wl.name}, K={wl.K}, R={wl.R}) in {el:.2f} s, fp64 numpy oracle; tokens/s "
              f"counts full-layer tokens ({mo} x {ro}/{wl.N} per step)")
    return n, el, n * mo * frac / el, sample


def format_bytes(N, K, keep):
    """Encoded size of a weight: bitmap, kept values and offset table (the 16-byte
    padding of each block, at most 14 bytes, left out)."""
    nb = (N // 128) * (K // 64)
    return N * K // 8 + 2 * N * keep + 4 * (nb + 1)


def l2_plan(wl):
    """Weight + adapter copies the timed loop rotates over so that no step finds its
    weights in L2: enough for twice the L2, at least 2, at most 64 (the smallest layer
    cannot outgrow the L2 this way; the config says so)."""
    keep = wl.K - int(np.floor(wl.sparsity * wl.K))
    per_copy = format_bytes(wl.N, wl.K, keep) + 2 * wl.R * (wl.K + wl.N)
    ncopies = min(64, max(2, int(np.ceil(2 * L2_BYTES / per_copy))))
    return ncopies, per_copy


def config_for(wl, M, ws):
    """The config block of the JSON line: the same for the CUDA arm and the reference arm."""
    ncopies, per_copy = l2_plan(wl)
    big = ncopies * per_copy > 2 * L2_BYTES
    return {"workload": f"{wl.name} N={wl.N} K={wl.K} R={wl.R} "
                        f"({'+'.join(str(r) for r in wl.ranks)}) M={M} sparsity={wl.sparsity:.6g}",
            "model": f"SALR linear layer ({wl.name} shape)", "global_batch": M * ws,
            "parallelism": f"replicas x{ws}",
            "l2": (f"inputs larger than L2: rotating {ncopies} weight+adapter copies "
                   f"({ncopies * per_copy / 2**20:.0f} MiB > 2x L2)" if big else
                   f"layer smaller than L2: rotating {ncopies} weight+adapter copies "
                   f"({ncopies * per_copy / 2**20:.0f} MiB, partly L2-resident)")}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    wl = workload()
    M = M_TOKENS
    mo, ro, frac = oracle_sample(wl, M)
    step = oracle_sample_fn(wl, mo, ro)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = args.steps * mo * frac / el
    cores = blas_threads()
    sample = (f"each step: {mo} of the {M} tokens x {ro} of the {wl.N} output rows, fp64 "
              f"numpy oracle; tokens/s counts full-layer tokens ({mo} x {ro}/{wl.N} per step)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_for(wl, M, ws),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# Linear layers of one decoder layer of a Llama3-8B-shaped model (out x in) and the
# model's other tensors, for the compressed-size report (the pages quote the model size
# of Llama3-8B before and after compression).
LLAMA3_8B_LINEARS = [("q_proj", 4096, 4096), ("k_proj", 1024, 4096), ("v_proj", 1024, 4096),
                     ("o_proj", 4096, 4096), ("gate_proj", 14336, 4096),
                     ("up_proj", 14336, 4096), ("down_proj", 4096, 14336)]
LLAMA3_8B_LAYERS = 32
LLAMA3_8B_OTHER_PARAMS = 2 * 128256 * 4096 + (2 * LLAMA3_8B_LAYERS + 1) * 4096  # emb, head, norms


def run_encode_report(args):
    """salr_encode throughput and the encoded size of every linear layer of a
    Llama3-8B-shaped model (synthetic N(0, 0.02) weights drawn on the device)."""
    import torch

    from sparse_rank_linear_b200.build import build
    import sparse_rank_linear_b200 as salr

    build()
    salr.load_library()
    s = float(np.float32(0.5 if SPARSITY is None else SPARSITY))
    peaks, peak_src = measured_peaks()
    gen = torch.Generator(device="cuda")
    rows, enc_bytes, dense_bytes = [], 0, 0
    for name, N, K in LLAMA3_8B_LINEARS:
        gen.manual_seed(N * 131 + K)
        W = (torch.randn(N, K, generator=gen, device="cuda") * 0.02).to(torch.bfloat16)
        salr.encode(W, s).free()  # warm
        ms, wall = [], []
        for _ in range(max(3, args.steps)):
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0 = time.perf_counter()
            e0.record()
            h = salr.encode(W, s)  # synchronous: returns with the weight encoded
            e1.record()
            torch.cuda.synchronize()
            wall.append(time.perf_counter() - t0)
            ms.append(e0.elapsed_time(e1))
            info = h.info()
            h.free()
        keep = K - int(np.floor(s * K))
        nb = (N // 128) * (K // 64)
        # closed form of the format size, up to the 16-byte padding of each block
        lo = N * K // 8 + 2 * N * keep + 4 * (nb + 1)
        assert info["nnz"] == N * keep and lo <= info["bytes"] <= lo + 14 * nb, info
        t = statistics.median(ms) * 1e-3
        moved = 2 * N * K + info["bytes"]  # W read once, the format written once
        rows.append({"layer": name, "N": N, "K": K, "encoded_bytes": info["bytes"],
                     "dense_bytes": 2 * N * K, "ratio": 2 * N * K / info["bytes"],
                     "encode_ms": t * 1e3, "encode_wall_ms": statistics.median(wall) * 1e3,
                     "w_gbs": 2 * N * K / t / 1e9, "hbm_frac": moved / t / 1e9 / peaks["hbm_gbs"]})
        enc_bytes += info["bytes"]
        dense_bytes += 2 * N * K
        del W
    L = LLAMA3_8B_LAYERS
    enc_t = sum(r["encode_ms"] for r in rows) * 1e-3
    other = 2 * LLAMA3_8B_OTHER_PARAMS
    line = {"metric": "SALR encode throughput (dense W bytes/s) and encoded size, "
                      "Llama3-8B-shaped linear layers", "value": dense_bytes / enc_t / 1e9,
            "unit": "GB/s", "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "sparsity": s, "steps": max(3, args.steps),
            "model": {"linear_dense_bytes": L * dense_bytes, "linear_encoded_bytes": L * enc_bytes,
                      "linear_ratio": dense_bytes / enc_bytes,
                      "whole_dense_bytes": L * dense_bytes + other,
                      "whole_encoded_bytes": L * enc_bytes + other,
                      "whole_ratio": (L * dense_bytes + other) / (L * enc_bytes + other),
                      "other_tensors": "embedding, lm_head and norms kept dense bf16",
                      "encode_seconds": L * enc_t},
            "peak_hbm_gbs": peaks["hbm_gbs"], "peak_source": peak_src, "layers": rows}
    print(json.dumps(line), flush=True)


def run_adapter_report(args):
    """salr_residual_adapter on the workload's W: time, fp32 FMA rate against the
    CUDA-core peak, and the residual energy it leaves against the pages' factor."""
    import torch

    from sparse_rank_linear_b200.build import build
    import sparse_rank_linear_b200 as salr

    build()
    salr.load_library()
    wl = workload()
    N, K = wl.N, wl.K
    r = wl.ranks[0]
    l = min(r + 16, 160, N, K)
    q = 2
    s = wl.sparsity
    w_bits = synth.weight(wl)
    W = torch.from_numpy(np.ascontiguousarray(w_bits).view(np.int16)).view(torch.bfloat16).cuda()
    h = salr.encode(W, s)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(0)
    omega = torch.randn(K, l, generator=gen, device="cuda", dtype=torch.float32)
    salr.residual_adapter(W, h, r, q=q, omega=omega)  # warm
    ms, wall = [], []
    for _ in range(max(3, args.steps)):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        e0.record()
        A, B, sig = salr.residual_adapter(W, h, r, q=q, omega=omega)  # synchronous
        e1.record()
        torch.cuda.synchronize()
        wall.append(time.perf_counter() - t0)
        ms.append(e0.elapsed_time(e1))
    # measurement only: the residual and the energy the adapter leaves, in fp32 torch
    E = W.float() - h.decode().float()
    total = float((E.double() ** 2).sum())
    err = float(((E - (A.float() @ B.float()).T).double() ** 2).sum())
    t = statistics.median(ms) * 1e-3
    lp = (l + 31) // 32 * 32
    flops = (4 + 4 * q) * N * K * l  # the E and E^T products (the dominant work)
    sm = torch.cuda.get_device_properties(0).multi_processor_count
    clk = max_sm_mhz() or 1965.0
    fp32_peak = sm * 128 * 2 * clk * 1e6 / 1e12
    line = {"metric": "SALR residual adapter build (randomized truncated SVD of W0 - W_hat)",
            "value": t * 1e3, "unit": "ms", "higher_is_better": False, "dtype": "f32",
            "data": "synthetic", "workload": f"{WORKLOAD} N={N} K={K} r={r} l={l} q={q} "
                                            f"sparsity={s:.6g}",
            "steps": max(3, args.steps), "wall_ms": statistics.median(wall) * 1e3,
            "roofline": {"bound": "alu", "achieved": flops / t / 1e12, "peak": fp32_peak,
                         "unit": "TFLOP/s", "frac": flops / t / 1e12 / fp32_peak,
                         "peak_source": f"{sm} SMs x 128 fp32 lanes x 2 x {clk:.0f} MHz",
                         "algorithmic_flops": flops, "padded_columns": lp},
            "residual_energy_left": err / total,
            "pages_factor_bound": 1.0 - r / min(N, K),
            "sigma_top": [float(x) for x in sig[:4].cpu()]}
    h.free()
    print(json.dumps(line), flush=True)


def traffic_for(kname, workload):
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kname}|{workload}")
    if not e or e.get("kernel_hash") != kernel_hash(kname):
        return None
    return e.get("bytes_per_launch")


# The (workload, tokens) points of the configurations; the headline line is the largest
# single-GPU one (large, 8192 tokens), the others are reported under "per_config".
POINTS = (("tiny", 16), ("q_proj", 1), ("q_proj", 16), ("up_proj", 2048), ("down_proj", 1),
          ("down_proj", 128), ("down_proj", 4096), ("large", 16), ("large", 8192))
# A timed region at least this long runs under the power cap: its tensor roofline is the
# sustained GEMM peak (a shorter region takes the burst peak).
LONG_REGION_MS = 500.0


class Layer:
    """One workload on the device: rotating encoded copies of W and adapter copies."""

    def __init__(self, salr, wl, dev):
        self.wl = wl
        self.w_bits = synth.weight(wl)
        ad = synth.adapters(wl)
        self.a_cat = np.concatenate([a for a, _ in ad], axis=1)
        self.b_cat = np.concatenate([b for _, b in ad], axis=0)
        W = dev(self.w_bits)
        self.ncopies, self.per_copy = l2_plan(wl)
        self.handles = [salr.encode(W, wl.sparsity) for _ in range(self.ncopies)]
        self.A = [dev(self.a_cat) for _ in range(self.ncopies)]
        self.B = [dev(self.b_cat) for _ in range(self.ncopies)]
        del W
        self.keep = wl.K - int(np.floor(wl.sparsity * wl.K))

    def free(self):
        for h in self.handles:
            h.free()
        self.handles, self.A, self.B = [], [], []


def roofline_of(wl, M, keep, kern_ms, region_ms, peaks, peak_src, traffic_key, plan):
    """The roofline block of one point: the bound (HBM bytes or tensor FLOPs, whichever
    takes longer at the measured peaks), achieved rate, fraction."""
    N, K, R = wl.N, wl.K, wl.R
    abytes = algorithmic_bytes(N, K, R, M, keep)
    aflops = algorithmic_flops(N, K, R, M)
    long_region = region_ms >= LONG_REGION_MS
    tpeak = peaks.get("bf16_tflops_sustained" if long_region else "bf16_tflops",
                      peaks["bf16_tflops"])
    t_hbm = abytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = aflops / (tpeak * 1e12)
    if t_hbm >= t_tc:
        achieved = abytes / (kern_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
        roof["peak_source"] = f"{peak_src} hbm_gbs"
    else:
        achieved = aflops / (kern_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tpeak, "unit": "TFLOP/s",
                "frac": achieved / tpeak}
        roof["peak_source"] = (f"{peak_src} "
                               f"{'bf16_tflops_sustained' if long_region else 'bf16_tflops'}"
                               f" ({'timed region of %.0f ms, under the power cap' % region_ms if long_region else 'short timed region: burst'})")
        roof["frac_of_burst_peak"] = achieved / peaks["bf16_tflops"]
    if M <= 64:
        kname = f"salr_stream_kernel<{16 if M <= 16 else 32 if M <= 32 else 64},20>"
    else:
        wide = int(plan.get("tile_rows", 128) == 256)
        kname = f"salr_prefill_kernel<{128 if M <= 128 else 256},{wide}>"
    roof["traffic"] = traffic_for(kname, traffic_key)
    roof["kernel"] = kname
    roof["kernels_per_call"] = plan["kernels"]
    roof["kernel_ms"] = kern_ms
    roof["algorithmic_bytes"] = abytes
    roof["algorithmic_flops"] = aflops
    return roof


def time_point(lib, salr, layer, M, steps, warmup, stream, ws, local):
    """K calls of the layer on device-resident inputs, back to back behind a GPU sleep
    (CUDA events at the two ends), then a diagnostic pass with an event pair around every
    call.  Returns the region's time (max over ranks), the per-call percentiles and the
    clocks seen."""
    import ctypes
    import torch
    import torch.distributed as dist

    wl = layer.wl
    X = torch.from_numpy(np.ascontiguousarray(synth.activations(wl, M)).view(np.int16)).view(
        torch.bfloat16).cuda()
    Y = torch.empty(M, wl.N, dtype=torch.bfloat16, device="cuda")
    sp = salr.binding._stream_ptr(stream)

    def launch(i):
        c = i % layer.ncopies
        rc = lib.salr_linear(ctypes.c_void_p(X.data_ptr()), M, layer.handles[c].handle,
                             ctypes.c_void_p(layer.A[c].data_ptr()),
                             ctypes.c_void_p(layer.B[c].data_ptr()), wl.R,
                             ctypes.c_void_p(Y.data_ptr()), sp)
        if rc:
            raise RuntimeError(salr.status_string(rc))

    # every copy is used once before timing (a handle allocates its scratch on first use)
    for i in range(max(warmup, layer.ncopies)):
        launch(i)
    torch.cuda.synchronize()
    if layer.handles[0].sync_status() != 0:
        raise RuntimeError("device status after warm-up")
    e_start = torch.cuda.Event(enable_timing=True)
    e_stop = torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        torch.cuda._sleep(int(2e9 * 40e-6 * steps) + 10_000_000)
        e_start.record(stream)
        for i in range(steps):
            launch(i)
        e_stop.record(stream)
        torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    total_ms = max_over_ranks(e_start.elapsed_time(e_stop), ws, "cuda")
    for h in layer.handles:
        status = h.sync_status()
        if status != 0:
            raise RuntimeError(f"device status {salr.status_string(status)}")
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    torch.cuda.synchronize()
    torch.cuda._sleep(int(2e9 * 40e-6 * steps) + 10_000_000)
    for i in range(steps):
        ev_s[i].record(stream)
        launch(i)
        ev_e[i].record(stream)
    torch.cuda.synchronize()
    per_launch = [ev_s[i].elapsed_time(ev_e[i]) for i in range(steps)]
    del X, Y
    return total_ms, per_launch, clocks.summary()


def time_e2e(lib, salr, layer, M, steps, warmup, stream, ws):
    """The same calls through salr_linear_host: pinned host activations in and host
    outputs back, the copies inside the timed region."""
    import ctypes
    import torch

    wl = layer.wl
    xh = torch.from_numpy(synth.activations(wl, M).view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = torch.empty(M, wl.N, dtype=torch.bfloat16).pin_memory()
    sp = salr.binding._stream_ptr(stream)
    # bounded so that the host copies of a prefill-sized step stay within a few seconds
    n = max(3, min(steps, int(4e9 // (2 * M * (wl.K + wl.N)))))

    def launch_host(i):
        c = i % layer.ncopies
        rc = lib.salr_linear_host(ctypes.c_void_p(xh.data_ptr()), M, layer.handles[c].handle,
                                  ctypes.c_void_p(layer.A[c].data_ptr()),
                                  ctypes.c_void_p(layer.B[c].data_ptr()), wl.R,
                                  ctypes.c_void_p(yh.data_ptr()), sp)
        if rc:
            raise RuntimeError(salr.status_string(rc))

    for i in range(warmup):
        launch_host(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    torch.cuda._sleep(int(2e9 * 60e-6 * n) + 10_000_000)
    e0.record(stream)
    for i in range(n):
        launch_host(i)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), ws, "cuda")
    return {"value": whole_job_rate(ws, n, M, ms), "unit": "tokens/s",
            "h2d_bytes_per_step": 2 * M * wl.K, "d2h_bytes_per_step": 2 * M * wl.N,
            "steps": n, "api": "salr_linear_host (pinned host X and Y)"}


def main():
    global WORKLOAD, M_TOKENS, SPARSITY
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--tokens", type=int, default=None,
                    help="M, tokens per call (default: the workload's largest)")
    ap.add_argument("--sparsity", type=float, default=None,
                    help="fraction of each row pruned (default: the workload's, 0.5)")
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["salr", "reference"], default="salr")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time the headline point only")
    ap.add_argument("--per-config-steps", type=int, default=100)
    ap.add_argument("--adapter-report", action="store_true",
                    help="time salr_residual_adapter on the workload's weight")
    ap.add_argument("--encode-report", action="store_true",
                    help="time salr_encode on Llama3-8B-shaped layers and report sizes")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    WORKLOAD, SPARSITY = args.workload, args.sparsity
    M_TOKENS = args.tokens if args.tokens is not None else max(synth.WORKLOADS[WORKLOAD].Ms)
    if SPARSITY is not None and not 0.0 <= SPARSITY < 1.0:
        ap.error("--sparsity must lie in [0, 1)")
    if args.impl == "reference":
        return run_reference(args)
    if args.encode_report:
        return run_encode_report(args)
    if args.adapter_report:
        return run_adapter_report(args)

    import torch
    import torch.distributed as dist

    from sparse_rank_linear_b200.build import build
    import sparse_rank_linear_b200 as salr

    ws, rank, local = dist_env()
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    if rank == 0:
        build()
    if ws > 1:
        dist.barrier()
    lib = salr.load_library()
    peaks, peak_src = measured_peaks()
    stream = torch.cuda.current_stream()

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()

    def traffic_key(wl):
        return wl.name if wl.sparsity == 0.5 else f"{wl.name} s={wl.sparsity:.6g}"

    def point_entry(layer, M, steps, region_ms, per_launch, clocks):
        wl = layer.wl
        plan = salr.plan(wl.N, wl.K, M, wl.R)
        kern_ms = region_ms / steps
        return {"workload": config_for(wl, M, ws)["workload"], "value": whole_job_rate(ws, steps, M, region_ms),
                "unit": "tokens/s", "steps": steps, "ms_per_step": kern_ms,
                "roofline": roofline_of(wl, M, layer.keep, kern_ms, region_ms, peaks, peak_src,
                                        traffic_key(wl), plan),
                "gpu_launches": steps * plan["kernels"],
                "per_launch_event_ms_p10_p50_p90": [float(np.percentile(per_launch, q))
                                                    for q in (10, 50, 90)],
                "clocks": clocks}

    # ---------------- headline point
    wl = workload()
    M = M_TOKENS
    layer = Layer(salr, wl, dev)
    torch.cuda.synchronize()
    total_ms, per_launch, clocks = time_point(lib, salr, layer, M, args.steps, args.warmup,
                                              stream, ws, local)
    head = point_entry(layer, M, args.steps, total_ms, per_launch, clocks)
    # context only: the same layer with a dense bf16 W through cuBLAS (torch),
    # Y = X W^T + (X A_cat) B_cat, the comparison the pages' speedup claim makes
    dense_ctx = dense_lora_context(layer.w_bits, synth.activations(wl, M), layer.a_cat,
                                   layer.b_cat, wl, M, args.steps, total_ms)
    e2e = time_e2e(lib, salr, layer, M, args.steps, args.warmup, stream, ws)
    line = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": config_for(wl, M, ws),
            "roofline": head["roofline"], "e2e": e2e,
            "gpu_launches": head["gpu_launches"], "clocks": clocks,
            "per_launch_event_ms_p10_p50_p90": head["per_launch_event_ms_p10_p50_p90"],
            "dense_lora_context": dense_ctx}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        n, el, rate, sample = time_oracle(wl, M)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": blas_threads(),
                                "kind": "oracle", "sample": sample}

    # ---------------- every configuration point, the same way (context for the headline)
    if not args.no_per_config and SPARSITY is None:
        per = []
        steps = min(args.steps, args.per_config_steps)
        cur = layer
        for name, Mp in POINTS:
            if cur is None or cur.wl.name != name:
                if cur is not None:
                    cur.free()
                    torch.cuda.synchronize()
                    torch.cuda.empty_cache()
                cur = Layer(salr, synth.WORKLOADS[name], dev)
                torch.cuda.synchronize()
            if cur is layer and Mp == M:
                e = dict(head)
                e["steps"] = args.steps
            else:
                t_ms, pl, ck = time_point(lib, salr, cur, Mp, steps, args.warmup, stream, ws, local)
                e = point_entry(cur, Mp, steps, t_ms, pl, ck)
            d = dense_lora_context(cur.w_bits, synth.activations(cur.wl, Mp), cur.a_cat,
                                   cur.b_cat, cur.wl, Mp, e["steps"], e["ms_per_step"] * e["steps"])
            e["dense_lora_ms_per_step"] = d["ms_per_step"]
            e["salr_speedup_vs_dense_lora"] = d["salr_speedup"]
            per.append(e)
        if cur is not None and cur is not layer:
            cur.free()
        line["per_config"] = per
    if rank == 0:
        print(json.dumps(line), flush=True)
    layer.free()
    if ws > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

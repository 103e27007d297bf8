#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200.

One step = one pass of the whole path over one batch: the fused forward
(O, LSE) followed by the recompute backward (preprocess, main, dQ finalize)
on the fwd+bwd workload: batch 1, 32 heads, Sq = Sk = 8192, head_dim 128,
causal, Q/K/V/dO i.i.d. N(0,1)*0.5 in bf16 (seeded, synthetic).

Throughput is attention TFLOP/s: forward 4*B*H*Sq*Sk*D (halved for causal)
plus backward 2.5x that (five products, one of them the recomputed scores).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun, one process per GPU; every rank processes its own
independent copy of the workload (weak scaling, no collective on the data
path); times are taken on the device and reduced with a max over ranks.
``--impl reference`` times the float64 CPU oracle (rank 0 only) on bounded
samples of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOPS at seq 8K–32K, D=128, bf16 vs B200 dense BF16 peak"
UNIT = "TFLOP/s"
WORKLOAD = dict(name="c5_b1h32s8192d128_fwdbwd", B=1, H=32, Hk=32, Sq=8192, Sk=8192, D=128,
                causal=1, win_left=-1, win_right=-1, input_scale=0.5, seed=1005)
# grouped K/V heads (GQA, 4 query heads per K/V head) at the same sizes
GQA_WORKLOAD = dict(name="gqa_b1h32hk8s8192d128_fwdbwd", B=1, H=32, Hk=8, Sq=8192, Sk=8192,
                    D=128, causal=1, win_left=-1, win_right=-1, input_scale=0.5, seed=1006)
# KV-cache decode: one new query row per sequence over a full 8192-row cache
DECODE_WORKLOAD = dict(name="decode_b8h32hk8l8192d128", B=8, Sq=1, H=32, Hk=8, Smax=8192,
                       D=128, causal=0, input_scale=0.5, seed=1007)
# the same step at head_dim 64 (the keys-on-lanes kernel with half-width K/V tiles,
# two CTAs per SM)
DECODE64_WORKLOAD = dict(name="decode_b8h32hk8l8192d64", B=8, Sq=1, H=32, Hk=8, Smax=8192,
                         D=64, causal=0, input_scale=0.5, seed=1010)
# four new rows per sequence (speculative steps) on one shared K/V head: 128 query rows per
# K/V head, so the rows-on-lanes decode kernel runs; a 32768-row cache (134 MB) exceeds L2
DECODE_ROWS_WORKLOAD = dict(name="decode_b8q4h32hk1l32768d128", B=8, Sq=4, H=32, Hk=1,
                            Smax=32768, D=128, causal=1, input_scale=0.5, seed=1017)
# packed variable-length batch: 32768 tokens in sequences of 128..4096 tokens
VARLEN_WORKLOAD = dict(name="varlen_t32768h32d128_fwdbwd", total=32768, len_lo=128,
                       len_hi=4096, H=32, Hk=32, D=128, causal=1, input_scale=0.5, seed=1008)
# padded batch: sequences of 128..4096 tokens (8192 in all) in (B, S, H, D) tensors with
# per-sequence lengths, S = the longest sequence
PADDED_WORKLOAD = dict(name="padded_t8192h32d128_fwdbwd", total=8192, len_lo=128,
                       len_hi=4096, H=32, Hk=32, D=128, causal=1, input_scale=0.5, seed=1016)
# head_dim 64 forward alone: B2 H32 S8192 causal (inputs 192 MiB, larger than L2)
FWD64_WORKLOAD = dict(name="fwd_b2h32s8192d64_causal", B=2, H=32, Hk=32, Sq=8192, Sk=8192,
                      D=64, causal=1, win_left=-1, win_right=-1, input_scale=0.5, seed=1011)
# head_dim 256: B1 H16 S8192 causal
D256_WORKLOAD = dict(name="fwd_b1h16s8192d256_causal", B=1, H=16, Hk=16, Sq=8192, Sk=8192,
                     D=256, causal=1, win_left=-1, win_right=-1, input_scale=0.5, seed=1009)
# forward alone on the attention configurations (name, B, H, S, causal, window, counted
# GFLOP: 4*B*H*S*S*D, halved for causal; the window row counts visible pairs only)
FWD_SWEEP = [
    ("c2_b2h16s2048d128_causal", 2, 16, 2048, 1, (-1, -1), 34.36),
    ("c3_b1h32s8192d128_causal", 1, 32, 8192, 1, (-1, -1), 549.76),
    ("c3_b1h32s8192d128", 1, 32, 8192, 0, (-1, -1), 1099.51),
    ("c4_b1h32s32768d128_causal", 1, 32, 32768, 1, (-1, -1), 8796.09),
    ("c4_b1h32s32768d128_window4096", 1, 32, 32768, 1, (4096, 0), 2062.09),
    ("b2h32s8192d64_causal", 2, 32, 8192, 1, (-1, -1), 549.76),
]
# the forward alone on the causal 7B-decoder-like layer (B1 H32 Sq=Sk=8192 D128,
# inputs N(0,1)*0.5), timed by itself inside the default run
C3_CAUSAL = dict(name="c3_b1h32s8192d128_causal_fwd", B=1, H=32, Hk=32, Sq=8192, Sk=8192,
                 D=128, causal=1, win_left=-1, win_right=-1, input_scale=0.5, seed=1003)
C3_LAUNCHES = 200
# the two small configurations the oracle finishes in full (forward)
ORACLE_FULL = [
    dict(name="c1_b1h2s128d64", B=1, H=2, Hk=2, Sq=128, Sk=128, D=64, causal=0, win_left=-1,
         win_right=-1, input_scale=1.0, seed=1001),
    dict(name="c2_b2h16s2048d128_causal", B=2, H=16, Hk=16, Sq=2048, Sk=2048, D=128, causal=1,
         win_left=-1, win_right=-1, input_scale=1.0, seed=1002),
]
WORKLOADS = {"fwdbwd": WORKLOAD, "gqa": GQA_WORKLOAD, "decode": DECODE_WORKLOAD,
             "decode64": DECODE64_WORKLOAD, "decoderows": DECODE_ROWS_WORKLOAD,
             "varlen": VARLEN_WORKLOAD, "padded": PADDED_WORKLOAD,
             "d256": D256_WORKLOAD, "d256fwd": D256_WORKLOAD,
             "fwd64": FWD64_WORKLOAD,
             "fwdsweep": None}
D256_FWD_METRIC = "attention fwd TFLOPS, head_dim 256, bf16 vs B200 dense BF16 peak"
FWD64_METRIC = "attention fwd TFLOPS, head_dim 64, bf16 vs B200 dense BF16 peak"
D256_METRIC = "attention fwd+bwd TFLOPS, head_dim 256, bf16 vs B200 dense BF16 peak"
DECODE_METRIC = "KV-cache decode: cached K/V bytes read per second"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0, "source": "fallback"}
BWD_KERNEL_SOURCES = ["bwd_sm100.cuh", "ptx.cuh", "common.cuh"]
FWD_KERNEL_SOURCES = ["fwd_sm100.cuh", "ptx.cuh", "common.cuh"]
BWD256_KERNEL_SOURCES = ["bwd256_sm100.cuh", "ptx.cuh", "ptx_d256.cuh", "common.cuh"]
FWD256_KERNEL_SOURCES = ["fwd256_sm100.cuh", "ptx.cuh", "common.cuh"]


def kernel_names(w):
    """(metric, forward kernel, its sources, backward main kernel, its sources) of a workload."""
    if w["D"] == 256:
        return (D256_METRIC, "attn_fwd_d256_kernel", FWD256_KERNEL_SOURCES,
                "attn_bwd_d256_kernel", BWD256_KERNEL_SOURCES)
    return (METRIC, f"attn_fwd_kernel<{w['D']}>", FWD_KERNEL_SOURCES,
            f"attn_bwd_main_kernel<{w['D']}>", BWD_KERNEL_SOURCES)
ORACLE_ROWS_PER_SAMPLE = 512


# ---------------------------------------------------------------------------
# work accounting
# ---------------------------------------------------------------------------
def fwd_flops(w) -> float:
    f = 4.0 * w["B"] * w["H"] * w["Sq"] * w["Sk"] * w["D"]
    return f / 2 if w["causal"] else f


def bwd_flops(w) -> float:
    return 2.5 * fwd_flops(w)


def step_flops(w) -> float:
    return fwd_flops(w) + bwd_flops(w)


def visible_keys(i, w) -> int:
    d = w["Sk"] - w["Sq"]
    lo, hi = 0, w["Sk"] - 1
    if w["causal"]:
        hi = min(hi, i + d)
    if w["win_left"] >= 0:
        lo = max(lo, i + d - w["win_left"])
    if w["win_right"] >= 0:
        hi = min(hi, i + d + w["win_right"])
    return max(0, hi - lo + 1)


# ---------------------------------------------------------------------------
# distributed plumbing (no collective touches attention data)
# ---------------------------------------------------------------------------
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate_value(per_rank_flops: float, n_ranks: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: all ranks' work over the slowest rank's time."""
    return per_rank_flops * n_ranks / (max_ms * 1e-3) / 1e12


def pipelined_e2e(device, stream, host_in, dev_sets, out_names, run, n_steps):
    """End-to-end milliseconds per step through the public API, fed the way a
    training or serving loop feeds a GPU: step i's inputs are copied from pinned
    host memory on one copy stream while step i-1 computes on `stream` and step
    i-2's results are copied back to pinned host memory on a second copy stream.
    Device inputs and outputs are double-buffered (`dev_sets`, two dicts of
    tensors); every step's host->device and device->host copies lie inside the
    timed region, which ends when the last results are in host memory.
    run(d) launches one step on `stream` reading and writing the tensors of d."""
    import torch
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    out_host = [{n: torch.empty(d[n].shape, dtype=d[n].dtype).pin_memory() for n in out_names}
                for d in dev_sets]
    ev = lambda: torch.cuda.Event()
    ev_in, ev_comp, ev_out = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def one(i):
        slot = i & 1
        d = dev_sets[slot]
        s_in.wait_stream(stream) if i == 0 else None
        if i >= 2:
            s_in.wait_event(ev_comp[slot])  # step i-2 has finished reading these inputs
        with torch.cuda.stream(s_in):
            for n, t in host_in.items():
                d[n].copy_(t, non_blocking=True)
        ev_in[slot].record(s_in)
        stream.wait_event(ev_in[slot])
        if i >= 2:
            stream.wait_event(ev_out[slot])  # step i-2's results have left these outputs
        run(d)
        ev_comp[slot].record(stream)
        s_out.wait_event(ev_comp[slot])
        with torch.cuda.stream(s_out):
            for n in out_names:
                out_host[slot][n].copy_(d[n], non_blocking=True)
        ev_out[slot].record(s_out)

    for i in range(2):  # warm-up of the copy streams and both buffer sets
        one(i)
    torch.cuda.synchronize(device)
    barrier(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    for i in range(n_steps):
        one(i)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    return reduce_max(e0.elapsed_time(e1), device) / n_steps


# ---------------------------------------------------------------------------
# peaks, clocks, committed ncu traffic
# ---------------------------------------------------------------------------
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS)


def sources_sha(files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "exact_attention_156_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


def traffic_key(kernel: str, w, fmt: str = "bf16") -> str:
    """Name of a kernel's line in profiles/traffic_per_launch.txt: the kernel for
    the headline workload in bf16, kernel@workload[/f16] for the others."""
    if w is WORKLOAD and fmt == "bf16":
        return kernel
    return f"{kernel}@{w['name']}" + ("/f16" if fmt == "f16" else "")


def committed_traffic(kernel: str, sha: str):
    """DRAM bytes per launch recorded from an ncu capture, if the kernel's
    sources have not changed since (profiles/traffic_per_launch.txt)."""
    path = os.path.join(ROOT, "profiles", "traffic_per_launch.txt")
    try:
        for line in open(path):
            parts = line.split()
            if len(parts) >= 3 and not line.startswith("#") and parts[0] == kernel:
                if parts[1] == sha:
                    return float(parts[2])
    except OSError:
        pass
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while it runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for r in rows for j in range(4) if r[5 + j] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle samples (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------
def oracle_sample_inputs(w):
    from synth import bf16_bits_to_f32, make_inputs
    bits = make_inputs(w["B"], w["Sq"], w["Sk"], w["H"], w["D"], w["seed"], w["input_scale"],
                       with_dout=True, Hk=w["Hk"])
    return {n: bf16_bits_to_f32(bits[n]) for n in ("q", "k", "v", "do")}


def oracle_sample(inputs, w, sample_idx: int):
    """fwd+bwd of the oracle for ORACLE_ROWS_PER_SAMPLE seeded query rows of
    one head (their O, LSE, dQ and their share of dK, dV).  Returns
    (seconds, attention flops of that sample by the metric's convention)."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(10_000 + sample_idx)
    h = int(rng.integers(0, w["H"]))
    rows = np.sort(rng.choice(w["Sq"], size=ORACLE_ROWS_PER_SAMPLE, replace=False))
    pairs = sum(visible_keys(int(i), w) for i in rows)
    t0 = time.perf_counter()
    oracle.attention_backward_rows(inputs["q"], inputs["k"], inputs["v"], inputs["do"], 0, h,
                                   rows, 1.0 / math.sqrt(w["D"]), w["causal"], w["win_left"],
                                   w["win_right"])
    dt = time.perf_counter() - t0
    return dt, 14.0 * w["D"] * pairs  # 4*D (fwd) + 10*D (bwd) per visible pair


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(w, budget_s: float = 15.0):
    inputs = oracle_sample_inputs(w)
    tot_s, tot_f, n = 0.0, 0.0, 0
    while tot_s < budget_s and n < 64:
        dt, fl = oracle_sample(inputs, w, n)
        tot_s += dt
        tot_f += fl
        n += 1
    value = tot_f / tot_s / 1e12
    return {"value": value, "unit": UNIT, "cores": blas_threads(),
            "kind": "oracle",
            # the whole workload at the sampled rate (extrapolated per visible pair)
            "extrapolated_full_step_s": step_flops(w) / (value * 1e12),
            "sample": f"{n} samples x {ORACLE_ROWS_PER_SAMPLE} seeded query rows of one head of "
                      f"{w['name']} (fwd O/LSE, bwd dQ rows and their dK/dV share), float64 numpy, "
                      f"{tot_s:.1f} s total; flops counted as 14*D per visible pair"}


def oracle_full_forward():
    """The oracle's forward over the two small configurations in full (every
    row of every head), each timed once; TFLOP/s by the metric's convention."""
    import oracle
    from synth import bits_to_f32, make_inputs
    out = []
    for w in ORACLE_FULL:
        bits = make_inputs(w["B"], w["Sq"], w["Sk"], w["H"], w["D"], w["seed"], w["input_scale"])
        x = {n: bits_to_f32(bits[n]) for n in ("q", "k", "v")}

        def timed():
            t0 = time.perf_counter()
            oracle.attention_forward(x["q"], x["k"], x["v"], 1.0 / math.sqrt(w["D"]),
                                     w["causal"])
            return time.perf_counter() - t0

        dt = timed()
        out.append({"workload": w["name"], "seconds": dt,
                    "tflops": fwd_flops(w) / dt / 1e12, "cores": blas_threads(),
                    "sample": "whole configuration, forward, float64 numpy"})
        if w["Sq"] * w["Sk"] * w["B"] * w["H"] <= 1 << 20:
            # the smallest configuration also on one host core
            try:
                from threadpoolctl import threadpool_limits
                with threadpool_limits(limits=1):
                    dt1 = timed()
                out.append({"workload": w["name"], "seconds": dt1,
                            "tflops": fwd_flops(w) / dt1 / 1e12, "cores": 1,
                            "sample": "whole configuration, forward, float64 numpy, one thread"})
            except ImportError:
                pass
    return out


def time_c3_causal_forward(device, stream, launches: int = C3_LAUNCHES, warmup: int = 5):
    """The causal forward of B1 H32 Sq=Sk=8192 D128 (inputs N(0,1)*0.5, 192 MiB,
    larger than L2) launched back to back, with its own clock samples."""
    import torch
    from exact_attention_156_b200 import attn_fwd, get_last_device_error
    from synth import make_inputs
    w = C3_CAUSAL
    bits = make_inputs(w["B"], w["Sq"], w["Sk"], w["H"], w["D"], w["seed"], w["input_scale"])
    q, k, v = (torch.from_numpy(bits[n].view("int16")).view(torch.bfloat16).to(device)
               for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((w["B"], w["H"], w["Sq"]), dtype=torch.float32, device=device)
    step = lambda: attn_fwd(q, k, v, causal=True, out=o, lse=lse, stream=stream)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(device).uuid))
    sampler.start()
    e0.record(stream)
    for _ in range(launches):
        step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    if get_last_device_error() != 0:
        raise RuntimeError("device-side error in the C3 causal forward")
    ms = e0.elapsed_time(e1) / launches
    peaks = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    tf = fwd_flops(w) / (ms * 1e-3) / 1e12
    del q, k, v, o, lse
    return {"workload": f"{w['name']}: forward alone, B=1 H=32 Sq=Sk=8192 D=128 causal bf16, "
                        f"inputs N(0,1)*0.5 (192 MiB, no L2 flush)",
            "kernel": "attn_fwd_kernel<128>", "launches": launches, "warmup": warmup,
            "ms": ms, "tflops": tf, "peak": peak, "frac": tf / peak,
            "peak_source": f"{peaks.get('source')} bf16_tflops (burst)", "clocks": clocks}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    inputs = oracle_sample_inputs(w)
    for i in range(args.warmup):
        oracle_sample(inputs, w, 1000 + i)
    tot_s, tot_f = 0.0, 0.0
    for i in range(args.steps):
        dt, fl = oracle_sample(inputs, w, i)
        tot_s += dt
        tot_f += fl
    value = tot_f / tot_s / 1e12
    line = {
        "impl": "reference", "metric": kernel_names(w)[0], "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_dict(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"each step: {ORACLE_ROWS_PER_SAMPLE} seeded query rows of one "
                                   f"head of {w['name']}, fwd+bwd in float64 numpy"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(w):
    heads = f"H={w['H']}" + (f" Hk={w['Hk']}" if w["Hk"] != w["H"] else "")
    in_mib = 2 * w["B"] * w["D"] * 2 * (w["Sq"] * w["H"] + w["Sk"] * w["Hk"]) / 2**20
    d = {"workload": f"{w['name']}: fwd+bwd, B={w['B']} {heads} Sq=Sk={w['Sq']} "
                     f"D={w['D']} causal bf16, inputs N(0,1)*{w['input_scale']}",
         "B": w["B"], "H": w["H"], "Sq": w["Sq"], "Sk": w["Sk"], "D": w["D"],
         "causal": bool(w["causal"]),
         "l2": f"no flush: inputs (Q,K,V,dO {in_mib:.0f} MiB) and outputs exceed the 126 MB L2"}
    if w["Hk"] != w["H"]:
        d["Hk"] = w["Hk"]
    return d


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_gpu(args):
    import torch
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(device)
    from exact_attention_156_b200 import (attn_bwd_stages, attn_bwd_workspace_size, attn_fwd,
                                          get_last_device_error)
    from synth import make_inputs

    w = WORKLOADS[args.workload]
    B, H, Sq, Sk, D = w["B"], w["H"], w["Sq"], w["Sk"], w["D"]
    causal = bool(w["causal"])
    win = (w["win_left"], w["win_right"])
    bits = make_inputs(B, Sq, Sk, H, D, w["seed"] + rank, w["input_scale"], with_dout=True,
                       Hk=w["Hk"], fmt=args.dtype)
    tdtype = torch.float16 if args.dtype == "f16" else torch.bfloat16
    host = {n: torch.from_numpy(bits[n].view("int16")).view(tdtype).pin_memory()
            for n in ("q", "k", "v", "do")}
    dev = {n: t.to(device) for n, t in host.items()}
    q, k, v, do = dev["q"], dev["k"], dev["v"], dev["do"]
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(attn_bwd_workspace_size(B, Sq, H, D), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    names = ["fwd", "bwd_preprocess", "bwd_main", "bwd_dq_finalize"]
    set0 = {"q": q, "k": k, "v": v, "do": do, "o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}

    def step(evs=None, d=set0):
        if evs is not None:
            evs[0].record(stream)
        attn_fwd(d["q"], d["k"], d["v"], causal=causal, window_size=win, out=d["o"],
                 lse=d["lse"], stream=stream)
        rec = (lambda i: evs[i + 1].record(stream)) if evs is not None else None
        attn_bwd_stages(d["q"], d["k"], d["v"], d["o"], d["do"], d["lse"], d["dq"], d["dk"],
                        d["dv"], ws, causal=causal, window_size=win, stream=stream, between=rec)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if get_last_device_error() != 0:
        raise RuntimeError("device-side timeout during warm-up")

    # timed region: K steps, per-kernel events on the launching stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(device).uuid))
    barrier(device)
    torch.cuda.synchronize(device)
    sampler.start()
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    clocks = sampler.stop()
    total_ms = start.elapsed_time(end)
    per_kernel = [statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps))
                  for j in range(4)]
    launches = 4 * args.steps
    if get_last_device_error() != 0:
        raise RuntimeError("device-side timeout during the timed region")
    max_ms = reduce_max(total_ms, device)
    ms_per_step = max_ms / args.steps
    value = aggregate_value(step_flops(w), world, ms_per_step)

    # end to end through the public API with host buffers: every step copies its
    # inputs (Q, K, V, dO) from pinned memory and its results (O, LSE, dQ, dK, dV)
    # back, pipelined across steps on two copy streams (pipelined_e2e)
    out_names = ("o", "lse", "dq", "dk", "dv")
    e2e_steps = max(3, min(args.steps, 10))
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(set0[n].numel() * set0[n].element_size() for n in out_names)

    e2e = None
    if not args.no_e2e:
        set1 = {n: torch.empty_like(t) for n, t in set0.items()}
        e2e_ms = pipelined_e2e(device, stream, host, [set0, set1], out_names,
                               lambda d: step(None, d), e2e_steps)
        if get_last_device_error() != 0:
            raise RuntimeError("device-side timeout during the end-to-end leg")
        e2e = {"value": aggregate_value(step_flops(w), world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "steps": e2e_steps,
               "pipelining": "inputs of step i copied in while step i-1 computes and step "
                             "i-2's results are copied out (two copy streams, double-buffered "
                             "device tensors); every step's copies inside the timed region"}

    c3 = None
    if args.workload == "fwdbwd" and args.dtype == "bf16" and not args.no_c3:
        barrier(device)
        c3 = time_c3_causal_forward(device, stream)
        launches += c3["launches"] + c3["warmup"]
        barrier(device)

    peaks = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    metric, fwd_name, fwd_src, bwd_name, bwd_src = kernel_names(w)
    bwd_main_tflops = bwd_flops(w) / (per_kernel[2] * 1e-3) / 1e12
    fwd_tflops = fwd_flops(w) / (per_kernel[0] * 1e-3) / 1e12
    kernels = {
        "fwd": {"ms": per_kernel[0], "tflops": fwd_tflops, "frac": fwd_tflops / peak},
        "bwd_preprocess": {"ms": per_kernel[1]},
        "bwd_main": {"ms": per_kernel[2], "tflops": bwd_main_tflops,
                     "frac": bwd_main_tflops / peak},
        "bwd_dq_finalize": {"ms": per_kernel[3]},
    }
    line = {
        "metric": metric, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
        "config": config_dict(w),
        "roofline": {"bound": "tensor", "kernel": bwd_name,
                     "achieved": bwd_main_tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": bwd_main_tflops / peak,
                     "peak_source": f"{peaks.get('source')} bf16_tflops (burst)",
                     "traffic": committed_traffic(traffic_key(bwd_name.split("<")[0], w, args.dtype),
                                                  sources_sha(bwd_src))},
        "kernels": kernels,
        "fwd_roofline": {"bound": "tensor", "kernel": fwd_name,
                         "achieved": fwd_tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": fwd_tflops / peak,
                         "traffic": committed_traffic(traffic_key(fwd_name.split("<")[0], w, args.dtype),
                                                      sources_sha(fwd_src))},
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if c3 is not None:
        line["fwd_c3_causal"] = c3
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
        if args.workload == "fwdbwd":
            line["cpu_baseline"]["full_configs"] = oracle_full_forward()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def decode_bytes(w) -> float:
    """Algorithmic HBM bytes of one decode call: every valid cached K and V
    element once, plus the query rows read and the output rows written."""
    kv = 2.0 * w["B"] * w["Smax"] * w["Hk"] * w["D"] * 2
    qo = 2.0 * w["B"] * w["Sq"] * w["H"] * w["D"] * 2
    return kv + qo


DECODE_KERNEL_SOURCES = ["decode_sm100.cuh", "ptx.cuh", "common.cuh"]


def decode_kernel_name(w) -> str:
    """The split kernel attn_decode runs for a workload: keys on the lanes with
    at most 16 query rows per K/V head, else rows on the lanes."""
    if (w["H"] // w["Hk"]) * w["Sq"] <= 16:
        return "attn_decode_t16_kernel"
    return "attn_decode_kernel"



def decode_oracle_inputs(w, rank: int = 0):
    from synth import bits_to_f32, make_inputs
    bits = make_inputs(w["B"], w["Sq"], w["Smax"], w["H"], w["D"], w["seed"] + rank,
                       w["input_scale"], Hk=w["Hk"])
    return {n: bits_to_f32(bits[n]) for n in ("q", "k", "v")}


def decode_oracle_step(inputs, w):
    """One oracle pass over the whole decode workload (every sequence, every
    head, full-length cache).  Returns its seconds."""
    import numpy as np
    import oracle
    t0 = time.perf_counter()
    oracle.attention_decode(inputs["q"], inputs["k"], inputs["v"],
                            np.full(w["B"], w["Smax"]), 1.0 / math.sqrt(w["D"]), w["causal"])
    return time.perf_counter() - t0


def decode_cpu_baseline(w, budget_s: float = 10.0):
    inputs = decode_oracle_inputs(w)
    tot, n = 0.0, 0
    while tot < budget_s and n < 64:
        tot += decode_oracle_step(inputs, w)
        n += 1
    return {"value": n * decode_bytes(w) / tot / 1e9, "unit": "GB/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{n} passes of the float64 numpy oracle over the whole {w['name']} "
                      f"workload ({tot:.1f} s total)"}


def decode_config(w):
    return {"workload": f"{w['name']}: decode, B={w['B']} Sq={w['Sq']} H={w['H']} Hk={w['Hk']} "
                        f"cache {w['Smax']} rows (all valid) D={w['D']}, inputs "
                        f"N(0,1)*{w['input_scale']}",
            "B": w["B"], "Sq": w["Sq"], "H": w["H"], "Hk": w["Hk"], "Smax": w["Smax"],
            "D": w["D"],
            "l2": f"no flush: the K/V cache ({decode_bytes(w) / 2**20:.0f} MiB) exceeds the "
                  "126 MB L2"}


def run_decode_reference(args):
    rank, _, _ = dist_env()
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    inputs = decode_oracle_inputs(w)
    for _ in range(args.warmup):
        decode_oracle_step(inputs, w)
    tot = sum(decode_oracle_step(inputs, w) for _ in range(args.steps))
    value = args.steps * decode_bytes(w) / tot / 1e9
    print(json.dumps({
        "impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": decode_config(w),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": blas_threads(),
                         "kind": "oracle",
                         "sample": f"each step: the whole {w['name']} workload, float64 numpy"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)
    return 0


def run_decode(args):
    """The KV-cache decode workload: the cache is resident on the device (it is
    the state a decode step reads); one call = split kernel + combine kernel."""
    import torch
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(device)
    from exact_attention_156_b200 import (attn_decode, attn_decode_workspace_size,
                                          get_last_device_error)
    from synth import make_inputs
    w = WORKLOADS[args.workload]
    B, Sq, H, Hk, Smax, D = w["B"], w["Sq"], w["H"], w["Hk"], w["Smax"], w["D"]
    bits = make_inputs(B, Sq, Smax, H, D, w["seed"] + rank, w["input_scale"], Hk=Hk,
                       fmt=args.dtype)
    tdtype = torch.float16 if args.dtype == "f16" else torch.bfloat16
    as_t = lambda a: torch.from_numpy(a.view("int16")).view(tdtype)
    q_host = as_t(bits["q"]).pin_memory()
    q = q_host.to(device)
    kc, vc = as_t(bits["k"]).to(device), as_t(bits["v"]).to(device)
    seqlens = torch.full((B,), Smax, dtype=torch.int32, device=device)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device=device)
    ws = torch.empty(attn_decode_workspace_size(B, Sq, Smax, H, Hk, D), dtype=torch.uint8,
                     device=device)
    stream = torch.cuda.current_stream(device)
    step = lambda: attn_decode(q, kc, vc, seqlens, causal=bool(w["causal"]), out=o, lse=lse,
                               workspace=ws, stream=stream)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    barrier(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(device).uuid))
    sampler.start()
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    clocks = sampler.stop()
    if get_last_device_error() != 0:
        raise RuntimeError("device-side timeout during the timed region")
    ms = reduce_max(start.elapsed_time(end), device) / args.steps
    gbs = world * decode_bytes(w) / (ms * 1e-3) / 1e9
    # end to end: the new query rows from pinned host memory, O and LSE back to the host
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    l_host = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    torch.cuda.synchronize(device)
    barrier(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        q.copy_(q_host, non_blocking=True)
        step()
        o_host.copy_(o, non_blocking=True)
        l_host.copy_(lse, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    e2e_ms = reduce_max(e0.elapsed_time(e1), device) / args.steps
    peaks = load_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    line = {
        "metric": DECODE_METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
        "config": decode_config(w),
        "roofline": {"bound": "hbm",
                     "kernel": f"{decode_kernel_name(w)} (timed with its combine launch)",
                     "achieved": decode_bytes(w) / (ms * 1e-3) / 1e9, "peak": peak,
                     "unit": "GB/s", "frac": decode_bytes(w) / (ms * 1e-3) / 1e9 / peak,
                     "peak_source": f"{peaks.get('source')} hbm_gbs",
                     "traffic": committed_traffic(traffic_key(decode_kernel_name(w), w,
                                                              args.dtype),
                                                  sources_sha(DECODE_KERNEL_SOURCES))},
        "e2e": {"value": world * decode_bytes(w) / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": q_host.numel() * q_host.element_size(),
                "d2h_bytes_per_step": o_host.numel() * o_host.element_size()
                + l_host.numel() * l_host.element_size(), "ms_per_step": e2e_ms},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = decode_cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def varlen_lengths(w):
    from synth import packed_lengths
    return packed_lengths(w["total"], w["len_lo"], w["len_hi"], w["seed"])


def varlen_fwd_flops(w, lengths) -> float:
    """4*D per (query, key) pair of each sequence, halved for causal (the
    headline's convention, per sequence)."""
    f = sum(4.0 * w["H"] * L * L * w["D"] for L in lengths)
    return f / 2 if w["causal"] else f


def varlen_config(w, lengths, padded=False):
    if padded:
        B, S = len(lengths), max(lengths)
        gb = 4 * B * S * w["H"] * w["D"] * 2 / 1e9
        return {"workload": f"{w['name']}: fwd+bwd of a padded batch (B={B}, S={S}, "
                            f"H={w['H']}, D={w['D']}) of {w['total']} real tokens in sequences "
                            f"of {min(lengths)}..{max(lengths)} (lengths log-uniform in "
                            f"[{w['len_lo']}, {w['len_hi']}]) with per-sequence lengths, causal, "
                            f"inputs N(0,1)*{w['input_scale']}, padding rows zero",
                "B": B, "S": S, "real_tokens": w["total"], "H": w["H"], "D": w["D"],
                "causal": bool(w["causal"]),
                "l2": f"no flush: inputs (Q,K,V,dO {gb:.2f} GB) exceed the 126 MB L2"}
    return {"workload": f"{w['name']}: fwd+bwd of a packed batch, {len(lengths)} sequences of "
                        f"{min(lengths)}..{max(lengths)} tokens ({w['total']} in all, lengths "
                        f"log-uniform in [{w['len_lo']}, {w['len_hi']}]), H={w['H']} "
                        f"D={w['D']} causal, inputs N(0,1)*{w['input_scale']}",
            "total_tokens": w["total"], "sequences": len(lengths), "H": w["H"], "D": w["D"],
            "causal": bool(w["causal"]),
            "l2": "no flush: inputs (Q,K,V,dO 256 MiB) and outputs exceed the 126 MB L2"}


def varlen_oracle_step(inputs, w, lengths, idx: int):
    """Oracle fwd+bwd of one head of one sequence of the batch (seeded pick).
    Returns (seconds, flops by the metric's convention)."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(20_000 + idx)
    b = int(rng.integers(0, len(lengths)))
    h = int(rng.integers(0, w["H"]))
    c0 = sum(lengths[:b])
    L = lengths[b]
    cu = [0, L]
    sl = lambda x: x[c0:c0 + L, h:h + 1]
    t0 = time.perf_counter()
    oracle.attention_backward_varlen(sl(inputs["q"]), sl(inputs["k"]), sl(inputs["v"]),
                                     sl(inputs["do"]), cu, cu, 1.0 / math.sqrt(w["D"]),
                                     w["causal"])
    dt = time.perf_counter() - t0
    return dt, 3.5 * 4.0 * L * L * w["D"] / (2 if w["causal"] else 1)


def varlen_oracle_inputs(w, rank: int = 0):
    from synth import bits_to_f32, make_inputs
    T = w["total"]
    bits = make_inputs(1, T, T, w["H"], w["D"], w["seed"] + rank, w["input_scale"],
                       with_dout=True, Hk=w["Hk"])
    return {n: bits_to_f32(bits[n])[0] for n in ("q", "k", "v", "do")}


def run_varlen_reference(args):
    rank, _, _ = dist_env()
    if rank != 0:
        return 0
    w = PADDED_WORKLOAD if args.workload == "padded" else VARLEN_WORKLOAD
    lengths = varlen_lengths(w)
    inputs = varlen_oracle_inputs(w)
    for i in range(args.warmup):
        varlen_oracle_step(inputs, w, lengths, 1000 + i)
    tot_s = tot_f = 0.0
    for i in range(args.steps):
        dt, fl = varlen_oracle_step(inputs, w, lengths, i)
        tot_s += dt
        tot_f += fl
    value = tot_f / tot_s / 1e12
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_s / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": varlen_config(w, lengths, args.workload == "padded"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"each step: fwd+bwd of one seeded (sequence, head) of "
                                   f"{w['name']}, float64 numpy"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)
    return 0


def run_varlen(args):
    """fwd + bwd of a packed variable-length batch (one step = both calls); with
    --workload padded, a smaller batch of such sequences in (B, S, H, D) tensors
    through attn_fwd_padded / attn_bwd_padded."""
    import numpy as np
    import torch
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(device)
    from exact_attention_156_b200 import (attn_bwd_padded, attn_bwd_padded_workspace_size,
                                          attn_bwd_varlen, attn_bwd_varlen_workspace_size,
                                          attn_fwd_padded, attn_fwd_padded_workspace_size,
                                          attn_fwd_varlen, get_last_device_error)
    from synth import make_inputs
    padded = args.workload == "padded"
    w = PADDED_WORKLOAD if padded else VARLEN_WORKLOAD
    lengths = varlen_lengths(w)
    T, H, D = w["total"], w["H"], w["D"]
    Bp, Lmax = len(lengths), max(lengths)
    bits = make_inputs(1, T, T, H, D, w["seed"] + rank, w["input_scale"], with_dout=True,
                       Hk=w["Hk"], fmt=args.dtype)
    tdtype = torch.float16 if args.dtype == "f16" else torch.bfloat16
    if padded:
        # sequence b's rows first in row block b, zeros after them
        starts = np.concatenate([[0], np.cumsum(lengths)])
        host = {}
        for n in ("q", "k", "v", "do"):
            a = np.zeros((Bp, Lmax, H, D), dtype=np.int16)
            for b, L in enumerate(lengths):
                a[b, :L] = bits[n][0][starts[b]:starts[b] + L].view(np.int16)
            host[n] = torch.from_numpy(a).view(tdtype).pin_memory()
        host["cu"] = torch.tensor(lengths, dtype=torch.int32).pin_memory()  # seqlens
    else:
        host = {n: torch.from_numpy(bits[n][0].view("int16")).view(tdtype).pin_memory()
                for n in ("q", "k", "v", "do")}
        cu_host = torch.from_numpy(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32))
        host["cu"] = cu_host.pin_memory()
    dev = {n: t.to(device) for n, t in host.items()}
    q, k, v, do, cu = dev["q"], dev["k"], dev["v"], dev["do"], dev["cu"]
    o = torch.empty_like(q)
    lse = torch.empty((Bp, H, Lmax) if padded else (H, T), dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if padded:
        ws_f = torch.empty(attn_fwd_padded_workspace_size(Bp, Lmax, Lmax, H, H, D),
                           dtype=torch.uint8, device=device)
        ws = torch.empty(attn_bwd_padded_workspace_size(Bp, Lmax, Lmax, H, H, D),
                         dtype=torch.uint8, device=device)
    else:
        ws = torch.empty(attn_bwd_varlen_workspace_size(Bp, T, H, D), dtype=torch.uint8,
                         device=device)
    stream = torch.cuda.current_stream(device)
    causal = bool(w["causal"])
    set0 = {"q": q, "k": k, "v": v, "do": do, "cu": cu, "o": o, "lse": lse, "dq": dq,
            "dk": dk, "dv": dv}

    def step(evs=None, d=set0):
        if evs is not None:
            evs[0].record(stream)
        if padded:
            attn_fwd_padded(d["q"], d["k"], d["v"], d["cu"], d["cu"], causal=causal, out=d["o"],
                            lse=d["lse"], workspace=ws_f, stream=stream)
        else:
            attn_fwd_varlen(d["q"], d["k"], d["v"], d["cu"], d["cu"], Lmax, Lmax, causal=causal,
                            out=d["o"], lse=d["lse"], stream=stream)
        if evs is not None:
            evs[1].record(stream)
        if padded:
            attn_bwd_padded(d["q"], d["k"], d["v"], d["o"], d["do"], d["lse"], d["cu"], d["cu"],
                            causal=causal, dq=d["dq"], dk=d["dk"], dv=d["dv"], workspace=ws,
                            stream=stream)
        else:
            attn_bwd_varlen(d["q"], d["k"], d["v"], d["o"], d["do"], d["lse"], d["cu"], d["cu"],
                            Lmax, Lmax, causal=causal, dq=d["dq"], dk=d["dk"], dv=d["dv"],
                            workspace=ws, stream=stream)
        if evs is not None:
            evs[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(device).uuid))
    barrier(device)
    torch.cuda.synchronize(device)
    sampler.start()
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    clocks = sampler.stop()
    if get_last_device_error() != 0:
        raise RuntimeError("device-side error during the timed region")
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    ms = reduce_max(start.elapsed_time(end), device) / args.steps
    ff = varlen_fwd_flops(w, lengths)
    value = world * 3.5 * ff / (ms * 1e-3) / 1e12
    out_names = ("o", "lse", "dq", "dk", "dv")
    e2e = None
    if not args.no_e2e:
        n_e2e = max(3, min(args.steps, 10))
        set1 = {n: torch.empty_like(t) for n, t in set0.items()}
        e2e_ms = pipelined_e2e(device, stream, host, [set0, set1], out_names,
                               lambda d: step(None, d), n_e2e)
        if get_last_device_error() != 0:
            raise RuntimeError("device-side error during the end-to-end leg")
        e2e = {"value": world * 3.5 * ff / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host.values()),
               "d2h_bytes_per_step": sum(set0[n].numel() * set0[n].element_size()
                                         for n in out_names),
               "ms_per_step": e2e_ms, "steps": n_e2e,
               "pipelining": "inputs of step i copied in while step i-1 computes and step "
                             "i-2's results are copied out (two copy streams, double-buffered "
                             "device tensors); every step's copies inside the timed region"}
    peaks = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    bwd_tf = 2.5 * ff / (bwd_ms * 1e-3) / 1e12
    fwd_tf = ff / (fwd_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
        "config": varlen_config(w, lengths, padded),
        "roofline": {"bound": "tensor",
                     "kernel": ("attn_bwd_padded (gathers, scans, preprocess + main + dQ "
                                "finalize, scatters)" if padded else
                                "attn_bwd_varlen (preprocess + main + dQ finalize launches)"),
                     "achieved": bwd_tf, "peak": peak, "unit": "TFLOP/s", "frac": bwd_tf / peak,
                     "peak_source": f"{peaks.get('source')} bf16_tflops (burst)",
                     "traffic": None},
        "kernels": {("fwd_padded" if padded else "fwd_varlen"):
                    {"ms": fwd_ms, "tflops": fwd_tf, "frac": fwd_tf / peak},
                    ("bwd_padded" if padded else "bwd_varlen"):
                    {"ms": bwd_ms, "tflops": bwd_tf, "frac": bwd_tf / peak}},
        "e2e": e2e,
        # padded: forward 2 scans + 3 gathers + kernel + 2 scatters; backward 2 scans +
        # 6 gathers + 3 kernels + 3 scatters
        "gpu_launches": (22 if padded else 4) * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inputs = varlen_oracle_inputs(w)
        tot_s = tot_f = 0.0
        n = 0
        while tot_s < 10.0 and n < 64:
            dt, fl = varlen_oracle_step(inputs, w, lengths, n)
            tot_s += dt
            tot_f += fl
            n += 1
        line["cpu_baseline"] = {"value": tot_f / tot_s / 1e12, "unit": UNIT,
                                "cores": blas_threads(), "kind": "oracle",
                                "sample": f"{n} seeded (sequence, head) pairs of {w['name']}, "
                                          f"fwd+bwd in float64 numpy, {tot_s:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_fwd_only(args):
    """Forward-only workloads (head_dim 256 or 64, the forward alone)."""
    import torch
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(device)
    from exact_attention_156_b200 import attn_fwd, get_last_device_error
    from synth import make_inputs
    w = WORKLOADS[args.workload]
    fwd_metric = D256_FWD_METRIC if w["D"] == 256 else FWD64_METRIC
    B, H, Sq, Sk, D = w["B"], w["H"], w["Sq"], w["Sk"], w["D"]
    bits = make_inputs(B, Sq, Sk, H, D, w["seed"] + rank, w["input_scale"], Hk=w["Hk"],
                       fmt=args.dtype)
    tdtype = torch.float16 if args.dtype == "f16" else torch.bfloat16
    host = {n: torch.from_numpy(bits[n].view("int16")).view(tdtype).pin_memory()
            for n in ("q", "k", "v")}
    dev = {n: t.to(device) for n, t in host.items()}
    q, k, v = dev["q"], dev["k"], dev["v"]
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    causal = bool(w["causal"])
    step = lambda: attn_fwd(q, k, v, causal=causal, out=o, lse=lse, stream=stream)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    barrier(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(device).uuid))
    sampler.start()
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    clocks = sampler.stop()
    if get_last_device_error() != 0:
        raise RuntimeError("device-side error during the timed region")
    ms = reduce_max(start.elapsed_time(end), device) / args.steps
    ff = fwd_flops(w)
    tf = ff / (ms * 1e-3) / 1e12
    e2e = None
    if not args.no_e2e:
        n_e2e = max(3, min(args.steps, 10))
        set0 = {"q": q, "k": k, "v": v, "o": o, "lse": lse}
        set1 = {n: torch.empty_like(t) for n, t in set0.items()}
        run = lambda d: attn_fwd(d["q"], d["k"], d["v"], causal=causal, out=d["o"],
                                 lse=d["lse"], stream=stream)
        e2e_ms = pipelined_e2e(device, stream, host, [set0, set1], ("o", "lse"), run, n_e2e)
        if get_last_device_error() != 0:
            raise RuntimeError("device-side timeout during the end-to-end leg")
        e2e = {"value": world * ff / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host.values()),
               "d2h_bytes_per_step": o.numel() * o.element_size() + lse.numel() * lse.element_size(),
               "ms_per_step": e2e_ms, "steps": n_e2e,
               "pipelining": "inputs of step i copied in while step i-1 computes and step "
                             "i-2's results are copied out (two copy streams, double-buffered "
                             "device tensors); every step's copies inside the timed region"}
    peaks = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    line = {
        "metric": fwd_metric, "value": world * tf, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
        "config": {"workload": f"{w['name']}: forward, B={B} H={H} Sq=Sk={Sq} D={D} causal, "
                               f"inputs N(0,1)*{w['input_scale']}", "B": B, "H": H, "Sq": Sq,
                   "Sk": Sk, "D": D, "causal": causal,
                   "l2": f"no flush: inputs (Q,K,V {3 * B * Sq * H * D * 2 / 2**20:.0f} MiB) "
                         "exceed the 126 MB L2"},
        "roofline": {"bound": "tensor",
                     "kernel": "attn_fwd_d256_kernel" if D == 256 else f"attn_fwd_kernel<{D}>",
                     "achieved": tf,
                     "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                     "peak_source": f"{peaks.get('source')} bf16_tflops (burst)",
                     "traffic": None},
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = fwd_oracle_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def fwd_oracle_sample(inputs, w, sample_idx: int):
    """Oracle forward of ORACLE_ROWS_PER_SAMPLE seeded query rows of one head.
    Returns (seconds, flops: 4*D per visible pair)."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(30_000 + sample_idx)
    h = int(rng.integers(0, w["H"]))
    rows = np.sort(rng.choice(w["Sq"], size=ORACLE_ROWS_PER_SAMPLE, replace=False))
    trip = np.stack([np.zeros_like(rows), np.full_like(rows, h), rows], axis=1)
    pairs = sum(visible_keys(int(i), w) for i in rows)
    t0 = time.perf_counter()
    oracle.attention_forward_rows(inputs["q"], inputs["k"], inputs["v"], trip,
                                  1.0 / math.sqrt(w["D"]), w["causal"], w["win_left"],
                                  w["win_right"])
    return time.perf_counter() - t0, 4.0 * w["D"] * pairs


def fwd_oracle_baseline(w, budget_s: float = 10.0):
    inputs = oracle_sample_inputs(w)
    tot_s = tot_f = 0.0
    n = 0
    while tot_s < budget_s and n < 64:
        dt, fl = fwd_oracle_sample(inputs, w, n)
        tot_s += dt
        tot_f += fl
        n += 1
    return {"value": tot_f / tot_s / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} samples x {ORACLE_ROWS_PER_SAMPLE} seeded query rows of one head of "
                      f"{w['name']}, forward in float64 numpy, {tot_s:.1f} s"}


def run_fwd_only_reference(args):
    rank, _, _ = dist_env()
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    inputs = oracle_sample_inputs(w)
    for i in range(args.warmup):
        fwd_oracle_sample(inputs, w, 1000 + i)
    tot_s = tot_f = 0.0
    for i in range(args.steps):
        dt, fl = fwd_oracle_sample(inputs, w, i)
        tot_s += dt
        tot_f += fl
    value = tot_f / tot_s / 1e12
    print(json.dumps({
        "impl": "reference",
        "metric": D256_FWD_METRIC if w["D"] == 256 else FWD64_METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_s / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w['name']}: forward, B={w['B']} H={w['H']} "
                               f"Sq=Sk={w['Sq']} D={w['D']} causal"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"each step: {ORACLE_ROWS_PER_SAMPLE} seeded query rows of one "
                                   f"head of {w['name']}, forward in float64 numpy"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)
    return 0


def run_fwd_sweep(args):
    """Forward alone on each attention configuration (one GPU; seeded inputs
    N(0,1)*0.5 drawn on the device; K launches after W warm-ups per config).
    One JSON line; `value` is the C3 causal forward."""
    import torch
    from exact_attention_156_b200 import attn_fwd, get_last_device_error
    rank, world, _ = dist_env()
    if world > 1:
        raise SystemExit("--workload fwdsweep runs on one GPU")
    peaks = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    gen = torch.Generator(device="cuda")
    rows = []
    for name, B, H, S, causal, win, gflop in FWD_SWEEP:
        gen.manual_seed(1000 + len(rows))
        D = 64 if name.endswith("d64_causal") else 128
        q, k, v = ((torch.randn(B, S, H, D, device="cuda", generator=gen) * 0.5).bfloat16()
                   for _ in range(3))
        o = torch.empty_like(q)
        lse = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
        step = lambda: attn_fwd(q, k, v, causal=bool(causal), window_size=win, out=o, lse=lse)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(0).uuid))
        sampler.start()
        e0.record()
        for _ in range(args.steps):
            step()
        e1.record()
        torch.cuda.synchronize()
        clocks = sampler.stop()
        if get_last_device_error() != 0:
            raise RuntimeError(f"device-side error in {name}")
        ms = e0.elapsed_time(e1) / args.steps
        tf = gflop / ms
        rows.append({"workload": name, "ms": ms, "tflops": tf, "frac": tf / peak,
                     "l2": "inputs exceed L2" if 3 * q.numel() * 2 > 126e6 else
                     "inputs fit in L2", "clocks": clocks})
        del q, k, v, o, lse
    head = rows[1]
    print(json.dumps({
        "metric": "attention forward TFLOP/s per configuration", "value": head["tflops"],
        "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": head["ms"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "forward alone on C2, C3 (causal, non-causal), C4 (causal, "
                               "window (4096, 0)); value = C3 causal"},
        "roofline": {"bound": "tensor", "kernel": "attn_fwd_kernel<128>",
                     "achieved": head["tflops"], "peak": peak, "unit": UNIT,
                     "frac": head["tflops"] / peak,
                     "peak_source": f"{peaks.get('source')} bf16_tflops (burst)",
                     "traffic": committed_traffic("attn_fwd_kernel",
                                                  sources_sha(FWD_KERNEL_SOURCES))},
        "configs": rows, "gpu_launches": len(FWD_SWEEP) * (args.steps + args.warmup)}),
        flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--dtype", choices=["bf16", "f16"], default="bf16",
                    help="element format of the 16-bit tensors (default bf16)")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="fwdbwd",
                    help="fwdbwd: the headline fwd+bwd workload (default); gqa: the same sizes "
                         "with 8 K/V heads for 32 query heads; decode: KV-cache decode "
                         "(B8 H32 Hk8, 8192 cached rows, one new row); varlen: a packed batch "
                         "of 32768 tokens in sequences of 128..4096; padded: 8192 tokens in such "
                         "sequences in (B, S, H, D) tensors with per-sequence lengths; d256: "
                         "head_dim 256 forward + "
                         "backward, B1 H16 S8192 causal; d256fwd: its forward alone; fwd64: the "
                         "head_dim 64 forward alone, B2 H32 S8192 causal; decode64: the decode "
                         "step at head_dim 64; decoderows: four new rows per sequence on one "
                         "K/V head (rows-on-lanes decode kernel); fwdsweep: the forward alone "
                         "on C2-C4")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the timed oracle sample (it adds ~15 s of CPU time)")
    ap.add_argument("--no-c3", action="store_true",
                    help="skip the standalone C3 causal forward leg of the default workload")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer end-to-end leg (fewer launches under a profiler)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload in ("decode", "decode64", "decoderows"):
        return run_decode_reference(args) if args.impl == "reference" else run_decode(args)
    if args.workload in ("varlen", "padded"):
        return run_varlen_reference(args) if args.impl == "reference" else run_varlen(args)
    if args.workload in ("d256fwd", "fwd64"):
        return run_fwd_only_reference(args) if args.impl == "reference" else run_fwd_only(args)
    if args.workload == "fwdsweep":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the forward sweep has no "
                              "oracle arm; the fwdbwd workload carries it"}))
            return 0
        return run_fwd_sweep(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())

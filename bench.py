#!/usr/bin/env python
"""Benchmark of the SmoothQuant W8A8 smoothed-linear path on B200.

Workload: the four OPT-6.7B linears (qkv 4096->12288, out 4096->4096,
fc1 4096->16384, fc2 16384->4096) in fp16, nn.Linear weight layout, M = 2048
prefill tokens and a calibration stream of 128 x 512 tokens per linear,
alpha = 0.5.  Inputs are seeded synthetic draws (N(0,1) activations with 1%
outlier channels x U(20,120), N(0,0.02) weights); the pages' WikiText-2
calibration set and checkpoints are not available.

One step = the whole path over one batch, for every linear:
  sq_calib_absmax (calibration stream) -> [all-reduce MAX across ranks]
  -> sq_smooth_quant_weight -> sq_quant_act (the M tokens) -> sq_w8a8_linear.
value = INT8 tensor-core operations of the step (2*M*N*K summed over the
linears and the ranks) / step time, in TOPS; each row is also reported
against its own roofline.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]
Multi-GPU: launched with torch.distributed.run, one rank per GPU (weak
scaling: every rank calibrates on and multiplies its own tokens).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

WORKLOAD = ("OPT-6.7B linears qkv 4096x12288, out 4096x4096, fc1 4096x16384, fc2 16384x4096; fp16; "
            "M=2048 tokens; calibration 128x512 tokens per linear; alpha=0.5; W [N,K]")
METRIC = "W8A8 smoothed linear TOPS & % INT8 tensor peak; act-quant GB/s % of HBM"
INT8_PER_BF16 = 2.0  # nominal dense INT8 / dense bf16 tensor throughput (4.5 / 2.25 PFLOP/s)
# Kernel launches of libsq per linear per step: calib 1, weight 4
# (zero fill, column max, smoothing factor, row quantizer), act-quant 1,
# linear 1.
LAUNCHES_PER_LINEAR = 7
WEIGHT_LAUNCHES = 4

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) measured with
# ncu on a smaller launch of the same kernel, as a ratio to that launch's
# algorithmic bytes; the bench scales it to its own per-launch bytes (the
# traffic of these streaming kernels grows in proportion to the bytes they
# stream).  Each entry is tied to a hash of the source text of the kernel
# and of its launcher (grid shape), as measured, and reported as null once
# either changes.
TRAFFIC = {
    # calibration 65536 x 4096 fp16: 536904192 + 3106048 bytes for
    # 536870912 + 32768 algorithmic bytes
    "absmax_cols_kernel": {"source": "sq_bw.cu", "functions": ("absmax_cols_kernel", "absmax_cols_t"),
                           "sha": "134a86d99ba523e4",
                           "ratio": (536904192 + 3106048) / (536870912 + 32768)},
}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def function_text(src: str, name: str) -> str:
    """Source text of the definition of function `name` in src: from the
    line that opens it (its template line, if any) to its closing brace."""
    i = 0
    while True:
        i = src.index(name + "(", i)
        body = src.index("{", i)
        if src.find(";", i, body) < 0:  # a definition, not a call or declaration
            break
        i += len(name)
    start = src.rfind("\n\n", 0, i) + 2
    depth, j = 0, body
    while True:
        if src[j] == "{":
            depth += 1
        elif src[j] == "}":
            depth -= 1
            if depth == 0:
                return src[start:j + 1]
        j += 1


def src_hash(name: str, functions) -> str:
    p = os.path.join(ROOT, "w8a8_post_quantization_channel_b200", "csrc", name)
    with open(p) as f:
        src = f.read()
    text = "\n".join(function_text(src, fn) for fn in functions)
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def traffic_for(kernel: str, algorithmic_bytes: float):
    """Per-launch DRAM bytes for a launch moving algorithmic_bytes, or None."""
    t = TRAFFIC.get(kernel)
    if not t or src_hash(t["source"], t["functions"]) != t["sha"]:
        return None
    return int(round(t["ratio"] * algorithmic_bytes))


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = (bus_id or "").lower()
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        mine = [r for r in self.rows if self.bus_id and r[0].lower().endswith(self.bus_id)]
        self.rows = mine or self.rows
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"], "samples": 0}

        def num(s):
            try:
                return float(s)
            except ValueError:
                return None
        sm = [num(r[1]) for r in self.rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in self.rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in self.rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows),
                "power_w_max": max((num(r[3]) or 0.0) for r in self.rows)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
class Layer:
    pass


def make_layers(rank: int, device: str, M: int, calib_tokens: int):
    from w8a8_post_quantization_channel_b200 import synth
    layers = []
    for i, (name, K, N) in enumerate(synth.OPT_6_7B):
        d = synth.opt67b_layer(i, M=M, calib_tokens=calib_tokens, seed=2000 + 1000 * rank, device=device)
        # every rank holds the same weights; tokens differ per rank
        d["w"] = synth.weights(K, N, 2000 + 10 * i + 2, torch.float16, "nk", device=device)
        L = Layer()
        L.name, L.K, L.N, L.M = name, K, N, M
        L.calib, L.x, L.w = d["calib"], d["x"], d["w"]
        L.amax = torch.zeros(K, device=device)
        L.wq = torch.empty(N, K, dtype=torch.int8, device=device)
        L.ws = torch.empty(N, device=device)
        L.s = torch.empty(K, device=device)
        L.inv = torch.empty(K, device=device)
        L.xq = torch.empty(M, K, dtype=torch.int8, device=device)
        L.xs = torch.empty(M, device=device)
        L.y = torch.empty(M, N, dtype=torch.float16, device=device)
        layers.append(L)
    return layers


def step(layers, sq, world: int, ev=None):
    """One pass of the whole path; ev: dict row -> list of (start, end) events."""
    from w8a8_post_quantization_channel_b200.dist import allreduce_amax

    def timed(row, fn):
        if ev is None:
            fn()
            return
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        ev.setdefault(row, []).append((a, b))

    for L in layers:
        L.amax.zero_()  # each step calibrates from scratch
        timed("calib", lambda: sq.sq_calib_absmax(L.calib, L.amax))
        if world > 1:
            allreduce_amax(L.amax)
        timed("weight", lambda: sq.sq_smooth_quant_weight(L.w, sq.SQ_W_NK, L.amax, 0.5, wq=L.wq, w_scale=L.ws,
                                                          smooth=L.s, inv_smooth=L.inv))
        timed("act", lambda: sq.sq_quant_act(L.x, L.inv, xq=L.xq, x_scale=L.xs))
        timed("linear", lambda: sq.sq_w8a8_linear(L.xq, L.xs, L.wq, L.ws, torch.float16, y=L.y))


def row_work(layers):
    """Algorithmic bytes / ops per step for each row (one rank)."""
    calib = sum(L.calib.shape[0] * L.K * 2 + 8 * L.K for L in layers)
    weight = sum(2 * L.N * L.K * 2 + L.N * L.K + 4 * L.N + 16 * L.K for L in layers)
    act = sum(L.M * L.K * 2 + L.M * L.K + 4 * L.M + 4 * L.K for L in layers)
    ops = sum(2 * L.M * L.N * L.K for L in layers)
    lin_bytes = sum(L.M * L.K + L.N * L.K + L.M * L.N * 2 + 4 * (L.M + L.N) for L in layers)
    return dict(calib=calib, weight=weight, act=act, linear_ops=ops, linear_bytes=lin_bytes)


def bench_ours(args, rank, world, local_rank):
    import torch.distributed as dist
    import w8a8_post_quantization_channel_b200 as sq

    device = f"cuda:{local_rank}"
    torch.cuda.set_device(local_rank)
    M, calib_tokens = 2048, 128 * 512
    layers = make_layers(rank, device, M, calib_tokens)
    work = row_work(layers)
    pk = peaks()
    torch.cuda.synchronize()

    props = torch.cuda.get_device_properties(local_rank)
    bus = f"{props.pci_domain_id:04x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
    clocks = ClockSampler(bus)
    clocks.start()
    for _ in range(args.warmup):
        step(layers, sq, world)
    if sq.sq_check_device_error() != sq.SQ_OK:
        raise RuntimeError("device-side timeout during warm-up")

    # -- timed region: K steps back to back ----------------------------------
    # (no events between the calls: an event between two kernels would undo
    # their programmatic dependent launch)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step(layers, sq, world)
    t1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = t0.elapsed_time(t1)
    if sq.sq_check_device_error() != sq.SQ_OK:
        raise RuntimeError("device-side timeout during the timed region")

    # -- per-row kernel times: the same steps again, each call bracketed by
    # CUDA events on the launching stream ----------------------------------
    ev = {}
    row_steps = min(args.steps, 50)
    for _ in range(row_steps):
        step(layers, sq, world, ev)
    torch.cuda.synchronize()
    if sq.sq_check_device_error() != sq.SQ_OK:
        raise RuntimeError("device-side timeout during the per-row pass")
    row_ms = {r: sum(a.elapsed_time(b) for a, b in v) / row_steps for r, v in ev.items()}

    if world > 1:
        t = torch.tensor([ms_total], device=device, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_total = float(t.item())
    ms_step = ms_total / args.steps
    value = work["linear_ops"] * world / (ms_step * 1e-3) / 1e12

    # -- per-row roofline ---------------------------------------------------------
    int8_peak_sus = pk["bf16_sus"] * INT8_PER_BF16
    int8_peak = pk["bf16"] * INT8_PER_BF16
    nlin = len(layers)
    rows = {}
    for r, key in (("calib", "calib"), ("weight", "weight"), ("act", "act")):
        gbs = work[key] / (row_ms[r] * 1e-3) / 1e9
        rows[r] = {"ms_per_step": round(row_ms[r], 4), "launches_per_step": nlin * (WEIGHT_LAUNCHES if r == "weight" else 1),
                   "algorithmic_bytes_per_step": work[key], "GB/s": round(gbs, 1),
                   "frac_of_hbm": round(gbs / pk["hbm"], 4)}
    tops = work["linear_ops"] / (row_ms["linear"] * 1e-3) / 1e12
    rows["linear"] = {"ms_per_step": round(row_ms["linear"], 4), "launches_per_step": nlin,
                      "ops_per_step": work["linear_ops"], "TOPS": round(tops, 1),
                      "frac_of_int8_peak_sustained": round(tops / int8_peak_sus, 4),
                      "frac_of_int8_peak_burst": round(tops / int8_peak, 4)}
    dominant = max(row_ms, key=row_ms.get)
    if dominant == "linear":
        roof = {"kernel": "w8a8_gemm_tc_kernel", "bound": "tensor", "achieved": round(tops, 1),
                "peak": round(int8_peak_sus, 1), "unit": "TFLOP/s", "frac": round(tops / int8_peak_sus, 4),
                "traffic": None,
                "peak_note": "INT8 = 2 x measured sustained bf16 (nominal dense ratio 4.5/2.25)"}
    else:
        per_launch_bytes = work[dominant] / (nlin * (WEIGHT_LAUNCHES if dominant == "weight" else 1))
        per_launch_ms = row_ms[dominant] / (nlin * (WEIGHT_LAUNCHES if dominant == "weight" else 1))
        kname = {"calib": "absmax_cols_kernel", "act": "quant_rows_kernel", "weight": "weight path"}[dominant]
        ach = per_launch_bytes / (per_launch_ms * 1e-3) / 1e9
        roof = {"kernel": kname, "bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm"], "unit": "GB/s",
                "frac": round(ach / pk["hbm"], 4), "traffic": traffic_for(kname, per_launch_bytes),
                "bytes_per_launch": int(per_launch_bytes)}
    roof["peak_source"] = f"{pk['src']} (MEASURED_PEAKS.json)" if pk["src"] == "measured" else "fallback"

    out = {"metric": METRIC, "value": round(value, 2), "unit": "TOPS", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "i8", "data": "synthetic",
           "config": {"workload": WORKLOAD, "global_batch": M * world, "seq_len": None,
                      "parallelism": f"dp{world}",
                      "l2": "inputs larger than L2: each step streams 3.8 GB of calibration tokens and 0.4 GB of "
                            "weights per rank"},
           "roofline": roof, "rows": rows, "rows_timing": f"per-call CUDA events over {row_steps} further steps",
           "gpu_launches": LAUNCHES_PER_LINEAR * nlin * args.steps}

    if not args.no_e2e:
        out["e2e"] = bench_e2e(args, layers, sq, world, work)
    clocks.stop()
    out["clocks"] = clocks.summary()
    if world > 1:
        dist.barrier()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(scale=args.cpu_sample_scale)
    return out


def bench_e2e(args, layers, sq, world, work):
    """Same metric through the public API with host buffers: every step copies
    its inputs from pinned host memory and reads Y back."""
    import torch.distributed as dist
    host = []
    for L in layers:
        h = dict(calib=torch.empty(L.calib.shape, dtype=L.calib.dtype, pin_memory=True),
                 w=torch.empty(L.w.shape, dtype=L.w.dtype, pin_memory=True),
                 x=torch.empty(L.x.shape, dtype=L.x.dtype, pin_memory=True),
                 y=torch.empty(L.y.shape, dtype=L.y.dtype, pin_memory=True))
        h["calib"].copy_(L.calib)
        h["w"].copy_(L.w)
        h["x"].copy_(L.x)
        host.append(h)
    h2d = sum(h["calib"].nbytes + h["w"].nbytes + h["x"].nbytes for h in host)
    d2h = sum(h["y"].nbytes for h in host)
    steps = max(1, min(args.steps, args.e2e_steps))

    def e2e_step():
        for L, h in zip(layers, host):
            L.calib.copy_(h["calib"], non_blocking=True)
            L.w.copy_(h["w"], non_blocking=True)
            L.x.copy_(h["x"], non_blocking=True)
        step(layers, sq, world)
        for L, h in zip(layers, host):
            h["y"].copy_(L.y, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        e2e_step()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    if world > 1:
        t = torch.tensor([ms], device=layers[0].x.device, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    ms_step = ms / steps
    return {"value": round(work["linear_ops"] * world / (ms_step * 1e-3) / 1e12, 3), "unit": "TOPS",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms_step, 3)}


# ---------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
_SAMPLE_CACHE = {}


def _sample_inputs(scale: float):
    """Seeded inputs of the bounded oracle sample (built once per scale)."""
    import numpy as np

    from w8a8_post_quantization_channel_b200 import synth
    if scale in _SAMPLE_CACHE:
        return _SAMPLE_CACHE[scale]
    sizes = dict(c_rows=max(8, int(512 * scale)), w_rows=max(8, int(256 * scale)), a_rows=max(2, int(16 * scale)),
                 g_rows=max(1, int(2 * scale)))
    per_layer = []
    for i, (name, K, N) in enumerate(synth.OPT_6_7B):
        o = synth.outliers(K, frac=0.01, mult=(20.0, 120.0), seed=2000 + 10 * i)
        per_layer.append(dict(
            K=K, N=N,
            calib=synth.activations(sizes["c_rows"], K, o, 7 + i, torch.float16).float().numpy(),
            x=synth.activations(max(sizes["a_rows"], sizes["g_rows"]), K, o, 11 + i, torch.float16).float().numpy(),
            w=synth.weights(K, sizes["w_rows"], 13 + i, torch.float16, "nk").float().numpy(),
            wq=np.random.default_rng(i).integers(-127, 128, (N, K), dtype=np.int8),
            dw=np.full(N, 1e-3, np.float32)))
    _SAMPLE_CACHE[scale] = (sizes, per_layer)
    return sizes, per_layer


def oracle_sample(scale: float):
    """Times the CPU oracle on a bounded sample of every row of the step and
    scales each part to the full workload.  Returns (seconds per full step,
    description).  Single-threaded C: cores = 1."""
    import oracle
    oracle.build()
    M, T = 2048, 128 * 512
    sz, layers = _sample_inputs(scale)
    c_rows, w_rows, a_rows, g_rows = sz["c_rows"], sz["w_rows"], sz["a_rows"], sz["g_rows"]
    total = 0.0
    for d in layers:
        K, N = d["K"], d["N"]
        t0 = time.perf_counter()
        amax = oracle.calib_absmax(d["calib"])
        t1 = time.perf_counter()
        wmax = oracle.weight_absmax(d["w"], oracle.LAYOUT_NK)
        s, inv = oracle.smooth_factor(amax, wmax, 0.5)
        oracle.smooth_quant_weight(d["w"], oracle.LAYOUT_NK, s)
        t2 = time.perf_counter()
        xq, dx = oracle.quant_act(d["x"], inv)
        t3 = time.perf_counter()
        acc = oracle.gemm_i8(xq[:g_rows], d["wq"])
        oracle.round_to(oracle.dequant(acc, dx[:g_rows], d["dw"]), "f16")
        t4 = time.perf_counter()
        a_done = xq.shape[0]
        total += (t1 - t0) * T / c_rows + (t2 - t1) * N / w_rows + (t3 - t2) * M / a_done + (t4 - t3) * M / g_rows
    desc = (f"oracle (plain C, 1 thread) per linear: calibration {c_rows} of {T} tokens, weight path {w_rows} output "
            f"channels, act-quant {max(a_rows, g_rows)} of {M} tokens, INT8 product + dequant {g_rows} of {M} token "
            f"rows x all N; each part scaled linearly to the full step")
    return total, desc


def cpu_baseline(scale: float):
    from w8a8_post_quantization_channel_b200 import synth
    secs, desc = oracle_sample(scale)
    ops = sum(2 * 2048 * N * K for _, K, N in synth.OPT_6_7B)
    return {"value": ops / secs / 1e12, "unit": "TOPS", "cores": 1, "kind": "oracle", "sample": desc,
            "seconds_per_step_extrapolated": round(secs, 2)}


def bench_reference(args, rank, world):
    from w8a8_post_quantization_channel_b200 import synth
    if rank != 0:
        return None
    scale = 0.25
    for _ in range(args.warmup):
        oracle_sample(scale)
    secs = []
    desc = ""
    for _ in range(args.steps):
        s, desc = oracle_sample(scale)
        secs.append(s)
    sec = statistics.mean(secs)
    ops = sum(2 * 2048 * N * K for _, K, N in synth.OPT_6_7B)
    value = ops / sec / 1e12
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
            # the same workload description as this bench's own arm at this N
            "config": {"workload": WORKLOAD, "global_batch": 2048 * world, "seq_len": None,
                       "parallelism": f"dp{world}"},
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": 1, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-sample-scale", type=float, default=24.0)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    args.steps = max(1, args.steps)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        out = bench_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device(f"cuda:{local_rank}"))
    out = bench_ours(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

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
against its own roofline.  Beside the step, the line carries the two numbers
the metric names as fields of their own (int8_linear, act_quant) and two more
sets of rows, each timed as back-to-back launches captured in a CUDA graph
over rotating inputs larger than L2:
  decode         the decode-shaped linears of a Llama-2-7B block (M = 1, 32)
                 and a Llama-2-70B block (M = 8), against HBM;
  act_quant_16k  act-quant of 16384-token bf16 batches (Student-t, 1%
                 outlier channels x100) at K = 4096, 7168, 8192, 28672.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]
  python bench.py --op OP --M M --K K --N N --dtype DT [--iters I] [--time]
  python bench.py --sweep NAME
Multi-GPU: launched with torch.distributed.run, one rank per GPU (weak
scaling: every rank calibrates on and multiplies its own tokens).  --op runs
one library call on one shape (for profilers); --sweep times a list of the
workloads' shapes, one JSON line each.
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


def row_graph_ms(layers, sq) -> dict:
    """Per-step time of each row, its calls (one per linear) replayed back to
    back from a CUDA graph.  The activation rows rotate over extra copies of
    the four inputs, so that the replayed inputs exceed 2 x L2 as the other
    rows' already do (3.8 GB of calibration tokens, 0.4 GB of weights, 0.26
    GB of codes and weights per step)."""
    out = {}
    calls = {"calib": [], "weight": [], "act": [], "linear": []}
    copies = []
    for L in layers:
        calls["calib"].append(lambda L=L: sq.sq_calib_absmax(L.calib, L.amax))
        calls["weight"].append(lambda L=L: sq.sq_smooth_quant_weight(L.w, sq.SQ_W_NK, L.amax, 0.5, wq=L.wq,
                                                                      w_scale=L.ws, smooth=L.s, inv_smooth=L.inv))
        calls["linear"].append(lambda L=L: sq.sq_w8a8_linear(L.xq, L.xs, L.wq, L.ws, torch.float16, y=L.y))
    act_bytes = sum(L.x.numel() * L.x.element_size() for L in layers)
    reps = max(1, -(-(2 * L2_BYTES + 1) // act_bytes))
    for _ in range(reps):
        for L in layers:
            x = L.x.clone()
            copies.append(x)
            calls["act"].append(lambda L=L, x=x: sq.sq_quant_act(x, L.inv, xq=L.xq, x_scale=L.xs))
    for row, cs in calls.items():
        secs, _ = graph_seconds_per_call(cs, min_calls=40, max_calls=400)
        out[row] = secs * len(layers) * 1e3
    del copies
    return out


def row_work(layers):
    """Algorithmic bytes / ops per step for each row (one rank)."""
    calib = sum(L.calib.shape[0] * L.K * 2 + 8 * L.K for L in layers)
    weight = sum(2 * L.N * L.K * 2 + L.N * L.K + 4 * L.N + 16 * L.K for L in layers)
    act = sum(L.M * L.K * 2 + L.M * L.K + 4 * L.M + 4 * L.K for L in layers)
    ops = sum(2 * L.M * L.N * L.K for L in layers)
    lin_bytes = sum(L.M * L.K + L.N * L.K + L.M * L.N * 2 + 4 * (L.M + L.N) for L in layers)
    return dict(calib=calib, weight=weight, act=act, linear_ops=ops, linear_bytes=lin_bytes)


def config_dict(world: int, M: int = 2048) -> dict:
    """The workload description, identical in both arms' lines."""
    return {"workload": WORKLOAD, "global_batch": M * world, "seq_len": None, "parallelism": f"dp{world}",
            "l2": "inputs larger than L2: each step streams 3.8 GB of calibration tokens and 0.4 GB of "
                  "weights per rank; the decode and act_quant_16k rows rotate over input copies of more than "
                  "2 x L2 in all"}


# ---------------------------------------------------------------------------
# rows timed as back-to-back launches in a CUDA graph
# ---------------------------------------------------------------------------
def graph_seconds_per_call(calls, min_calls: int = 50, max_calls: int = 2000, bytes_per_call: float = 0.0):
    """Device time per call of `calls` (zero-argument launches), captured once
    in a CUDA graph and replayed back to back on the current stream between
    two CUDA events (no host launch cost, no event between the calls)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for c in calls:  # first calls outside the capture: per-device set-up
            c()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for c in calls:
            c()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    want = max_calls if bytes_per_call <= 0 else int(min(max_calls, max(min_calls, 2e10 / bytes_per_call)))
    reps = max(3, -(-want // len(calls)))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    secs = a.elapsed_time(b) * 1e-3 / (reps * len(calls))
    del g
    return secs, reps * len(calls)


L2_BYTES = 126 * 2 ** 20


def decode_rows(sq, pk, device):
    """Decode-shaped linears (M <= 64) of a Llama-2-7B block at M = 1 and 32
    (also with q|k|v and gate|up each stored as one matrix) and of a
    Llama-2-70B block at M = 8, bf16 out: each shape's launches
    rotate over copies of its Wq whose total exceeds 2 x L2, so every launch
    streams its weights from HBM.  Bytes per launch: N*K (Wq) + M*K + 2*M*N
    + 4*(M+N); fraction of the measured HBM copy bandwidth."""
    from w8a8_post_quantization_channel_b200 import synth
    out, blocks = [], {}
    cases = [("llama2-7b", M, sh) for M in (1, 32) for sh in synth.LLAMA2_7B]
    cases += [("llama2-70b", 8, sh) for sh in synth.LLAMA2_70B]
    # the same 7B block with its input-sharing projections stored as one
    # matrix each (q|k|v: 4096 -> 12288, gate|up: 4096 -> 22016), as serving
    # stacks lay them out: the same bytes in four launches instead of seven
    fused = [("qkv", 4096, 12288), ("o", 4096, 4096), ("gate_up", 4096, 22016), ("down", 11008, 4096)]
    cases += [("llama2-7b-fused", M, sh) for M in (1, 32) for sh in fused]
    for model, M, (name, K, N) in cases:
        g = synth.gen(7000 + K + N + M, device)
        copies = max(2, -(-(2 * L2_BYTES + 1) // (N * K)))
        wqs = [torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8, device=device) for _ in range(copies)]
        xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8, device=device)
        xs = torch.rand(M, generator=g, device=device) * 1e-2
        ws = torch.rand(N, generator=g, device=device) * 1e-2
        ys = [torch.empty(M, N, dtype=torch.bfloat16, device=device) for _ in range(copies)]
        need = sq.sq_w8a8_linear_workspace_size(M, N, K)
        work = torch.zeros(max(need, 1), dtype=torch.uint8, device=device)
        calls = [(lambda w=w, y=y: sq.sq_w8a8_linear(xq, xs, w, ws, torch.bfloat16, y=y, workspace=work))
                 for w, y in zip(wqs, ys)]
        nbytes = N * K + M * K + 2 * M * N + 4 * (M + N)
        secs, n = graph_seconds_per_call(calls, bytes_per_call=nbytes)
        gbs = nbytes / secs / 1e9
        out.append({"model": model, "linear": name, "M": M, "K": K, "N": N, "us": round(secs * 1e6, 2),
                    "GB/s": round(gbs, 1), "frac_of_hbm": round(gbs / pk["hbm"], 4), "launches_timed": n})
        key = f"{model}_M{M}"
        b = blocks.setdefault(key, [0, 0.0])
        b[0] += nbytes
        b[1] += secs
        del wqs, ys, work, calls
        torch.cuda.empty_cache()
    summary = {k: {"us_per_block": round(v[1] * 1e6, 2), "GB/s": round(v[0] / v[1] / 1e9, 1),
                   "frac_of_hbm": round(v[0] / v[1] / 1e9 / pk["hbm"], 4)} for k, v in blocks.items()}
    return {"method": "back-to-back launches in a CUDA graph, Wq rotating over copies > 2 x L2; bf16 out",
            "blocks": summary, "rows": out}


def act16k_rows(sq, pk, device):
    """sq_quant_act on 16384-token bf16 batches of Student-t(3) activations
    with 1% outlier channels x100, K = 4096, 7168, 8192, 28672; launches
    rotate over input copies whose total exceeds 2 x L2.  Bytes per launch:
    2 read + 1 written per element, 4 per token and per channel."""
    from w8a8_post_quantization_channel_b200 import synth
    rows = []
    M = 16384
    for K in (4096, 7168, 8192, 28672):
        o = synth.outliers(K, frac=0.01, mult=100.0, seed=K)
        copies = max(1, -(-(2 * L2_BYTES + 1) // (M * K * 2)))
        xs_in = [synth.activations(M, K, o, 8000 + K + i, torch.bfloat16, "student_t3", device=device)
                 for i in range(copies)]
        inv = torch.rand(K, generator=synth.gen(K, device), device=device) + 0.5
        xq = torch.empty(M, K, dtype=torch.int8, device=device)
        xsc = torch.empty(M, device=device)
        calls = [(lambda x=x: sq.sq_quant_act(x, inv, xq=xq, x_scale=xsc)) for x in xs_in]
        nbytes = M * K * 3 + 4 * (M + K)
        secs, n = graph_seconds_per_call(calls, bytes_per_call=nbytes)
        gbs = nbytes / secs / 1e9
        rows.append({"M": M, "K": K, "us": round(secs * 1e6, 2), "GB/s": round(gbs, 1),
                     "frac_of_hbm": round(gbs / pk["hbm"], 4), "launches_timed": n})
        del xs_in, xq, calls
        torch.cuda.empty_cache()
    return {"method": "back-to-back launches in a CUDA graph over input copies > 2 x L2", "rows": rows}


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
    row_ms_isolated = {r: sum(a.elapsed_time(b) for a, b in v) / row_steps for r, v in ev.items()}
    # -- and each row's calls back to back, as they run inside a step (a CUDA
    # graph per row, replayed; no event between the calls) ------------------
    row_ms = row_graph_ms(layers, sq)
    if sq.sq_check_device_error() != sq.SQ_OK:
        raise RuntimeError("device-side timeout during the per-row graphs")

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
           "config": config_dict(world, M),
           "roofline": roof,
           "int8_linear": {"TOPS": rows["linear"]["TOPS"],
                           "frac_of_int8_peak_burst": rows["linear"]["frac_of_int8_peak_burst"],
                           "frac_of_int8_peak_sustained": rows["linear"]["frac_of_int8_peak_sustained"],
                           "shapes": "OPT-6.7B qkv, out, fc1, fc2 at M = 2048, fp16 out",
                           "peak_note": "INT8 = 2 x measured bf16 (nominal dense ratio 4.5/2.25)"},
           "act_quant": {"GB/s": rows["act"]["GB/s"], "frac_of_hbm": rows["act"]["frac_of_hbm"],
                         "shapes": "2048 tokens x K = 4096 (x3), 16384 (x1), fp16"},
           "rows": rows,
           "rows_timing": "each row's calls for the four linears captured in a CUDA graph and replayed back to back "
                          "(inputs rotate over copies larger than 2 x L2), CUDA events around the replays",
           "rows_isolated_ms_per_step": {r: round(v, 4) for r, v in row_ms_isolated.items()},
           "rows_isolated_timing": f"each call bracketed by CUDA events, {row_steps} further steps",
           "gpu_launches": LAUNCHES_PER_LINEAR * nlin * args.steps}
    if not args.no_extra_rows:
        out["decode"] = decode_rows(sq, pk, device)
        out["act_quant_16k"] = act16k_rows(sq, pk, device)
        if sq.sq_check_device_error() != sq.SQ_OK:
            raise RuntimeError("device-side timeout in the decode or act_quant_16k rows")

    if not args.no_e2e:
        out["e2e"] = bench_e2e(args, layers, sq, world, work)
    clocks.stop()
    out["clocks"] = clocks.summary()
    if world > 1:
        dist.barrier()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(scale=args.cpu_sample_scale, procs=args.oracle_procs or host_cores())
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
GEMM_COLS = 1024  # output channels of the INT8-product sample (scaled to N)


def _sample_inputs(scale: float, seed: int = 0):
    """Seeded inputs of the bounded oracle sample (built once per process)."""
    import numpy as np

    from w8a8_post_quantization_channel_b200 import synth
    key = (scale, seed)
    if key in _SAMPLE_CACHE:
        return _SAMPLE_CACHE[key]
    sizes = dict(c_rows=max(8, int(512 * scale)), w_rows=max(8, int(256 * scale)), a_rows=max(2, int(16 * scale)),
                 g_rows=max(1, int(8 * scale)))
    per_layer = []
    for i, (name, K, N) in enumerate(synth.OPT_6_7B):
        o = synth.outliers(K, frac=0.01, mult=(20.0, 120.0), seed=2000 + 10 * i)
        s0 = 100 * seed
        per_layer.append(dict(
            K=K, N=N,
            calib=synth.activations(sizes["c_rows"], K, o, s0 + 7 + i, torch.float16).float().numpy(),
            x=synth.activations(max(sizes["a_rows"], sizes["g_rows"]), K, o, s0 + 11 + i,
                                torch.float16).float().numpy(),
            w=synth.weights(K, sizes["w_rows"], s0 + 13 + i, torch.float16, "nk").float().numpy(),
            wq=np.random.default_rng(seed * 10 + i).integers(-127, 128, (min(N, GEMM_COLS), K), dtype=np.int8),
            dw=np.full(min(N, GEMM_COLS), 1e-3, np.float32)))
    _SAMPLE_CACHE[key] = (sizes, per_layer)
    return sizes, per_layer


def oracle_sample(scale: float, seed: int = 0):
    """Times the CPU oracle (one thread, as it stands) on a bounded sample of
    every row of the step and scales each part to the full workload.
    Returns (seconds per full step on one core, description)."""
    import oracle
    oracle.build()
    M, T = 2048, 128 * 512
    sz, layers = _sample_inputs(scale, seed)
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
        cols = d["wq"].shape[0]
        total += ((t1 - t0) * T / c_rows + (t2 - t1) * N / w_rows + (t3 - t2) * M / a_done
                  + (t4 - t3) * (M / g_rows) * (N / cols))
    desc = (f"oracle (plain C, one thread per process) per linear: calibration {c_rows} of {T} tokens, weight path "
            f"{w_rows} output channels, act-quant {max(a_rows, g_rows)} of {M} tokens, INT8 product + dequant "
            f"{g_rows} of {M} token rows x {GEMM_COLS} output channels; each part scaled linearly to the full step")
    return total, desc


def _oracle_worker(task):
    scale, seed = task
    return oracle_sample(scale, seed)


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class OraclePool:
    """One process per host core (spawned, so that no CUDA state is
    inherited), each running the unmodified single-threaded oracle on its own
    sample at the same time as the others; the full step split over the
    processes then takes (mean per-process seconds per step) / processes."""

    def __init__(self, procs: int):
        import multiprocessing as mp
        self.procs = max(1, procs)
        self.pool = mp.get_context("spawn").Pool(self.procs)

    def step_seconds(self, scale: float, seed: int = 0):
        res = self.pool.map(_oracle_worker, [(scale, seed * self.procs + i) for i in range(self.procs)],
                            chunksize=1)
        return statistics.mean(r[0] for r in res) / self.procs, res[0][1]

    def close(self):
        self.pool.close()
        self.pool.join()


def _ops_per_step() -> int:
    from w8a8_post_quantization_channel_b200 import synth
    return sum(2 * 2048 * N * K for _, K, N in synth.OPT_6_7B)


def cpu_baseline(scale: float, procs: int):
    pool = OraclePool(procs)
    try:
        pool.step_seconds(min(scale, 1.0))  # process start-up and first builds, untimed
        secs, desc = pool.step_seconds(scale, seed=1)
    finally:
        pool.close()
    return {"value": _ops_per_step() / secs / 1e12, "unit": "TOPS", "cores": pool.procs, "kind": "oracle",
            "sample": f"{pool.procs} processes at once, each: {desc}",
            "seconds_per_step_extrapolated": round(secs, 3), "nproc": os.cpu_count(), "cpu_model": cpu_model()}


def bench_reference(args, rank, world):
    if rank != 0:
        return None
    scale = 0.5
    pool = OraclePool(args.oracle_procs or host_cores())
    try:
        for i in range(args.warmup):
            pool.step_seconds(scale, seed=i)
        secs, desc = [], ""
        for i in range(args.steps):
            s, desc = pool.step_seconds(scale, seed=args.warmup + i)
            secs.append(s)
    finally:
        pool.close()
    sec = statistics.mean(secs)
    value = _ops_per_step() / sec / 1e12
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
            "ms_per_step_kind": "extrapolated: each step times a bounded sample of the workload on every process "
                                "and scales it to the full step",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
            "config": config_dict(world),
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": pool.procs, "kind": "oracle",
                             "sample": f"{pool.procs} processes at once, each: {desc}", "nproc": os.cpu_count(),
                             "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------
# one library call on one shape (--op), or a sweep of the workloads' shapes
# (--sweep): for profilers and for the per-shape tables.  With --time (implied
# by --sweep) every iteration is timed with CUDA events on the launching
# stream, a 512 MB buffer is read between iterations so that L2 (126 MB)
# holds none of the operands (a read leaves clean lines behind, so the timed
# kernel pays no write-back of someone else's dirty data), and the median is
# reported against the measured peaks: algorithmic bytes / time against HBM
# for calib, act, weight and decode-shaped linears (M <= 64: streaming Wq
# dominates), 2MNK / time against the INT8 tensor peak (2 x measured bf16)
# otherwise.  Inputs are seeded device-side draws of the workloads'
# distributions.
# ---------------------------------------------------------------------------
DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
ESZ = {"f32": 4, "f16": 2, "bf16": 2}


def sweeps():
    from w8a8_post_quantization_channel_b200 import synth
    return {
        # decode-shaped linears: Llama-2-70B and -7B layers at M in {1, 8, 32, 64}
        "decode": [("linear", M, K, N, "bf16") for (K, N) in ((8192, 8192), (8192, 1024), (8192, 28672),
                                                                 (28672, 8192), (4096, 4096), (4096, 11008),
                                                                 (11008, 4096))
                   for M in (1, 8, 32, 64)],
        # activation quantization on 16384-token batches
        "act": [("act", 16384, K, 0, "bf16") for K in (4096, 7168, 8192, 28672)] + [("act", 2048, 4096, 0, "f16"),
                                                                                       ("act", 2048, 16384, 0, "f16")],
        # calibration chunks of the token stream
        "calib": [("calib", 131072, K, 0, "bf16") for K in (4096, 7168, 8192)] + [("calib", 32768, 28672, 0, "bf16"),
                                                                                     ("calib", 65536, 4096, 0, "f16"),
                                                                                     ("calib", 65536, 16384, 0, "f16")],
        # smoothing + weight quantization, [K, K] and the OPT shapes
        "weight": [("weight", 0, K, K, "bf16") for K in (4096, 7168, 8192, 28672)] + [("weight", 0, 4096, 12288, "f16"),
                                                                                         ("weight", 0, 16384, 4096, "f16")],
        # upstream producers (RMSNorm or LayerNorm + smoothing + per-token INT8)
        # and the static per-tensor quantizer on 16384-token batches
        "producer": [("rmsnorm", 16384, K, 0, "bf16") for K in (4096, 8192)] + [("rmsnorm", 2048, 4096, 0, "f16")]
                    + [("layernorm", 16384, K, 0, "bf16") for K in (4096, 8192)]
                    + [("layernorm", 2048, 4096, 0, "f16"), ("layernorm", 16384, 4096, 0, "f16")]
                    + [("static", 16384, K, 0, "bf16") for K in (4096, 8192)],
        # butterfly-rotated activation quantization (N = the rotation's block size n)
        "rot": [("rot", 16384, 4096, n, "bf16") for n in (16, 64, 256, 1024, 4096)] + [("rot", 16384, 8192, 256, "bf16"),
                                                                                        ("rot", 16384, 8192, 8192, "bf16")],
        # FP8 (E4M3): activation quantization, weight path, prefill and decode linears
        "fp8": [("act8", 16384, 4096, 0, "bf16"), ("weight8", 0, 8192, 8192, "bf16")]
               + [("linear8", 2048, K, N, "f16") for _, K, N in synth.OPT_6_7B]
               + [("linear8", 4096, K, N, "bf16") for _, K, N in synth.LLAMA2_70B[3:]]
               + [("linear8", M, 8192, 28672, "bf16") for M in (1, 16, 64)],
        # prefill-shaped linears
        "prefill": [("linear", 2048, K, N, "f16") for _, K, N in synth.OPT_6_7B]
                   + [("linear", 4096, K, N, "bf16") for _, K, N in synth.LLAMA2_70B[1:]]
                   + [("linear", M, 4096, 11008, "bf16") for M in (128, 1024, 4096)],
    }


def make_case(op, M, K, N, dtype, dev="cuda"):
    import w8a8_post_quantization_channel_b200 as sq
    from w8a8_post_quantization_channel_b200 import synth
    dt = DT[dtype]
    o = synth.outliers(K, frac=0.01, mult=100.0, seed=1)
    if op in ("rmsnorm", "layernorm", "static"):
        x = synth.activations(M, K, o, 2, dt, device=dev)
        inv = torch.rand(K, device=dev) + 0.5
        gamma = torch.rand(K, device=dev) + 0.5
        xq = torch.empty(M, K, dtype=torch.int8, device=dev)
        xs = torch.empty(M, device=dev)
        delta = torch.full((1,), 0.05, device=dev)
        nbytes = M * K * (ESZ[dtype] + 1) + 4 * (M + K)
        if op == "rmsnorm":
            gs = sq.sq_fold_smooth_into_norm(gamma, inv)
            return (lambda: sq.sq_rmsnorm_quant_act(x, gs, 1e-5, xq=xq, x_scale=xs)), nbytes, None
        if op == "layernorm":
            gs = sq.sq_fold_smooth_into_norm(gamma, inv)
            bs = sq.sq_fold_smooth_into_norm(torch.rand(K, device=dev) - 0.5, inv)
            return (lambda: sq.sq_layernorm_quant_act(x, gs, bs, 1e-5, xq=xq, x_scale=xs)), nbytes + 4 * K, None
        return (lambda: sq.sq_quant_act_static(x, inv, delta, xq=xq, x_scale=xs)), nbytes, None
    if op in ("calib", "act"):
        x = synth.activations(M, K, o, 2, dt, device=dev)
        amax = torch.zeros(K, device=dev)
        inv = torch.rand(K, device=dev) + 0.5
        xq = torch.empty(M, K, dtype=torch.int8, device=dev)
        xs = torch.empty(M, device=dev)
        if op == "calib":
            return (lambda: sq.sq_calib_absmax(x, amax)), M * K * ESZ[dtype] + 8 * K, None
        return (lambda: sq.sq_quant_act(x, inv, xq=xq, x_scale=xs)), M * K * (ESZ[dtype] + 1) + 4 * (M + K), None
    if op == "rot":
        x = synth.activations(M, K, o, 2, dt, device=dev)
        inv = torch.rand(K, device=dev) + 0.5
        n = N or 256
        L = n.bit_length() - 1
        theta = torch.rand(L, n // 2, generator=synth.gen(5, dev), device=dev) * 6.2831853
        cs = torch.stack([torch.cos(theta), torch.sin(theta)], dim=-1).contiguous()
        xq = torch.empty(M, K, dtype=torch.int8, device=dev)
        xs = torch.empty(M, device=dev)
        return (lambda: sq.sq_quant_act_rotated(x, inv, n, cs, xq=xq, x_scale=xs)), M * K * (ESZ[dtype] + 1) + 4 * (
            M + K), None
    if op == "act8":
        x = synth.activations(M, K, o, 2, dt, device=dev)
        inv = torch.rand(K, device=dev) + 0.5
        xq = torch.empty(M, K, dtype=torch.uint8, device=dev)
        xs = torch.empty(M, device=dev)
        return (lambda: sq.sq_quant_act_e4m3(x, inv, xq=xq, x_scale=xs)), M * K * (ESZ[dtype] + 1) + 4 * (M + K), None
    if op == "weight":
        w = synth.weights(K, N, 3, dt, "nk", device=dev)
        amax = torch.rand(K, device=dev) * 10
        outs = dict(wq=torch.empty(N, K, dtype=torch.int8, device=dev), w_scale=torch.empty(N, device=dev),
                    smooth=torch.empty(K, device=dev), inv_smooth=torch.empty(K, device=dev))
        fn = lambda: sq.sq_smooth_quant_weight(w, sq.SQ_W_NK, amax, 0.5, **outs)  # noqa: E731
        return fn, 2 * N * K * ESZ[dtype] + N * K + 4 * N + 16 * K, None
    if op == "weight8":
        w = synth.weights(K, N, 3, dt, "nk", device=dev)
        amax = torch.rand(K, device=dev) * 10
        outs = dict(wq=torch.empty(N, K, dtype=torch.uint8, device=dev), w_scale=torch.empty(N, device=dev),
                    smooth=torch.empty(K, device=dev), inv_smooth=torch.empty(K, device=dev))
        fn = lambda: sq.sq_smooth_quant_weight_e4m3(w, sq.SQ_W_NK, amax, 0.5, **outs)  # noqa: E731
        return fn, 2 * N * K * ESZ[dtype] + N * K + 4 * N + 16 * K, None
    if op == "linear8":
        g = synth.gen(4, dev)
        # E4M3 codes of N(0,1) draws scaled to use the format's range
        xq = (torch.randn(M, K, generator=g, device=dev) * 60).clamp(-448, 448).to(torch.float8_e4m3fn).view(
            torch.uint8)
        wq = (torch.randn(N, K, generator=g, device=dev) * 60).clamp(-448, 448).to(torch.float8_e4m3fn).view(
            torch.uint8)
        xs = torch.rand(M, device=dev) * 1e-2
        ws = torch.rand(N, device=dev) * 1e-2
        y = torch.empty(M, N, dtype=dt, device=dev)
        need = sq.sq_w8a8_linear_workspace_size(M, N, K)
        work = torch.zeros(max(need, 1), dtype=torch.uint8, device=dev) if need else None
        fn = lambda: sq.sq_w8a8_linear_e4m3(xq, xs, wq, ws, dt, y=y, workspace=work)  # noqa: E731
        return fn, M * K + N * K + M * N * ESZ[dtype] + 4 * (M + N), 2 * M * N * K
    g = synth.gen(4, dev)
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8, device=dev)
    wq = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8, device=dev)
    xs = torch.rand(M, device=dev) * 1e-2
    ws = torch.rand(N, device=dev) * 1e-2
    y = torch.empty(M, N, dtype=dt, device=dev)
    need = sq.sq_w8a8_linear_workspace_size(M, N, K)
    work = torch.zeros(max(need, 1), dtype=torch.uint8, device=dev) if need else None
    fn = lambda: sq.sq_w8a8_linear(xq, xs, wq, ws, dt, y=y, workspace=work)  # noqa: E731
    return fn, M * K + N * K + M * N * ESZ[dtype] + 4 * (M + N), 2 * M * N * K


def time_case(op, M, K, N, dtype, iters):
    import w8a8_post_quantization_channel_b200 as sq
    fn, nbytes, ops = make_case(op, M, K, N, dtype)
    flush = torch.ones(128 * 2 ** 20, dtype=torch.float32, device="cuda")  # 512 MB
    fn()
    torch.cuda.synchronize()
    times = []
    for i in range(iters):
        flush.sum()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) * 1e-3)
    if sq.sq_check_device_error() != sq.SQ_OK:
        raise SystemExit("device-side timeout")
    t = statistics.median(times)
    pk = peaks()
    hbm, int8_peak, src = pk["hbm"], INT8_PER_BF16 * pk["bf16"], pk["src"]
    out = {"op": op, "M": M, "K": K, "N": N, "dtype": dtype, "us": round(t * 1e6, 2),
           "GB/s": round(nbytes / t / 1e9, 1), "frac_hbm": round(nbytes / t / 1e9 / hbm, 3)}
    if ops is not None:
        out["TOPS"] = round(ops / t / 1e12, 1)
        # the FP8 and INT8 dense peaks are both 2 x bf16 (4.5 vs 2.25 PFLOP/s nominal)
        out["frac_fp8_peak" if op == "linear8" else "frac_int8_peak"] = round(ops / t / 1e12 / int8_peak, 3)
        out["bound"] = "hbm" if M <= 64 else "tensor"
    else:
        out["bound"] = "hbm"
    out["peaks"] = src
    return out


def run_cases(a):
    import w8a8_post_quantization_channel_b200 as sq
    if a.sweep:
        for case in sweeps()[a.sweep]:
            print(json.dumps(time_case(*case, iters=max(a.iters, 5))), flush=True)
            torch.cuda.empty_cache()
        return
    if a.time:
        print(json.dumps(time_case(a.op, a.M, a.K, a.N, a.dtype, a.iters)))
        return
    fn, _, _ = make_case(a.op, a.M, a.K, a.N, a.dtype)
    for _ in range(a.iters):
        fn()
    torch.cuda.synchronize()
    if sq.sq_check_device_error() != sq.SQ_OK:
        raise SystemExit("device-side timeout")
    print(f"case {a.op} M={a.M} K={a.K} N={a.N} {a.dtype} x{a.iters}: ok")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-rows", action="store_true", help="skip the decode and act_quant_16k rows")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-sample-scale", type=float, default=24.0)
    ap.add_argument("--oracle-procs", type=int, default=0, help="oracle processes (default: one per host core)")
    ap.add_argument("--op", choices=["calib", "weight", "act", "linear", "rmsnorm", "layernorm", "static", "act8",
                                     "weight8", "linear8", "rot"], help="run one library call on one shape")
    ap.add_argument("--sweep", help="time a list of the workloads' shapes (see sweeps())")
    ap.add_argument("--M", type=int, default=2048)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--N", type=int, default=4096)
    ap.add_argument("--dtype", choices=["f32", "f16", "bf16"], default="f16")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--time", action="store_true")
    args = ap.parse_args()
    if args.op or args.sweep:
        run_cases(args)
        return
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

"""Runs (and optionally times) one libsq operation on one shape, or a sweep
of the workloads' shapes, for profilers and roofline measurements.

  python -m w8a8_post_quantization_channel_b200.profile_case --op linear \
      --M 2048 --K 4096 --N 16384 --dtype f16 --iters 3
  python -m w8a8_post_quantization_channel_b200.profile_case --sweep decode

--op is calib (T = M tokens), weight (W [N, K]), act, rmsnorm and
layernorm (the fused norm producers), static (static-scale quantizer), linear, or the FP8 (E4M3)
forms act8, weight8 and linear8, or rot (butterfly-rotated act-quant, --N =
the rotation block size).  With
--time (implied by --sweep) every iteration is timed with CUDA events on
the launching stream, a 512 MB buffer is read between iterations so that
L2 (126 MB) holds none of the operands (a read leaves clean lines behind, so
the timed kernel pays no write-back of someone else's dirty data), and the
median is reported
against the measured peaks: algorithmic bytes / time against HBM for calib,
act, weight and decode-shaped linears (M <= 64: streaming Wq dominates),
2MNK / time against the INT8 tensor peak (2 x measured bf16) otherwise.
Inputs are seeded device-side draws of the benchmark's distributions.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics

import torch

import w8a8_post_quantization_channel_b200 as sq
from w8a8_post_quantization_channel_b200 import synth

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
ESZ = {"f32": 4, "f16": 2, "bf16": 2}
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SWEEPS = {
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


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), 2.0 * float(d["bf16_tflops"]), "measured"
    return 6650.0, 2.0 * 1590.0, "fallback"


def make_case(op, M, K, N, dtype, dev="cuda"):
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
    hbm, int8_peak, src = peaks()
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=["calib", "weight", "act", "linear", "rmsnorm", "layernorm", "static", "act8",
                                     "weight8", "linear8", "rot"])
    ap.add_argument("--sweep", choices=sorted(SWEEPS))
    ap.add_argument("--M", type=int, default=2048)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--N", type=int, default=4096)
    ap.add_argument("--dtype", choices=list(DT), default="f16")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--time", action="store_true")
    a = ap.parse_args()
    if a.sweep:
        for case in SWEEPS[a.sweep]:
            print(json.dumps(time_case(*case, iters=max(a.iters, 5))), flush=True)
            torch.cuda.empty_cache()
        return
    if a.op is None:
        raise SystemExit("--op or --sweep is required")
    if a.time:
        print(json.dumps(time_case(a.op, a.M, a.K, a.N, a.dtype, a.iters)))
        return
    fn, _, _ = make_case(a.op, a.M, a.K, a.N, a.dtype)
    for _ in range(a.iters):
        fn()
    torch.cuda.synchronize()
    if sq.sq_check_device_error() != sq.SQ_OK:
        raise SystemExit("device-side timeout")
    print(f"profile_case {a.op} M={a.M} K={a.K} N={a.N} {a.dtype} x{a.iters}: ok")


if __name__ == "__main__":
    main()

"""Runs one libsq operation on one shape a few times, for profilers.

  python -m w8a8_post_quantization_channel_b200.profile_case --op linear \
      --M 2048 --K 4096 --N 16384 --dtype f16 --iters 3

Inputs are seeded device-side draws of the benchmark's distributions;
--op is calib (T=M tokens), weight (W [N,K]), act or linear.
"""
from __future__ import annotations

import argparse

import torch

import w8a8_post_quantization_channel_b200 as sq
from w8a8_post_quantization_channel_b200 import synth

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=["calib", "weight", "act", "linear"], required=True)
    ap.add_argument("--M", type=int, default=2048)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--N", type=int, default=4096)
    ap.add_argument("--dtype", choices=list(DT), default="f16")
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args()
    dev = "cuda"
    dt = DT[a.dtype]
    o = synth.outliers(a.K, frac=0.01, mult=100.0, seed=1)
    if a.op in ("calib", "act"):
        x = synth.activations(a.M, a.K, o, 2, dt, device=dev)
        amax = torch.zeros(a.K, device=dev)
        inv = torch.rand(a.K, device=dev) + 0.5
        xq = torch.empty(a.M, a.K, dtype=torch.int8, device=dev)
        xs = torch.empty(a.M, device=dev)
        fn = (lambda: sq.sq_calib_absmax(x, amax)) if a.op == "calib" else \
            (lambda: sq.sq_quant_act(x, inv, xq=xq, x_scale=xs))
    elif a.op == "weight":
        w = synth.weights(a.K, a.N, 3, dt, "nk", device=dev)
        amax = torch.rand(a.K, device=dev) * 10
        outs = dict(wq=torch.empty(a.N, a.K, dtype=torch.int8, device=dev), w_scale=torch.empty(a.N, device=dev),
                    smooth=torch.empty(a.K, device=dev), inv_smooth=torch.empty(a.K, device=dev))
        fn = lambda: sq.sq_smooth_quant_weight(w, sq.SQ_W_NK, amax, 0.5, **outs)  # noqa: E731
    else:
        g = synth.gen(4, dev)
        xq = torch.randint(-127, 128, (a.M, a.K), generator=g, dtype=torch.int8, device=dev)
        wq = torch.randint(-127, 128, (a.N, a.K), generator=g, dtype=torch.int8, device=dev)
        xs = torch.rand(a.M, device=dev) * 1e-2
        ws = torch.rand(a.N, device=dev) * 1e-2
        y = torch.empty(a.M, a.N, dtype=dt, device=dev)
        fn = lambda: sq.sq_w8a8_linear(xq, xs, wq, ws, dt, y=y)  # noqa: E731
    for _ in range(a.iters):
        fn()
    torch.cuda.synchronize()
    if sq.sq_check_device_error() != sq.SQ_OK:
        raise SystemExit("device-side timeout")
    print(f"profile_case {a.op} M={a.M} K={a.K} N={a.N} {a.dtype} x{a.iters}: ok")


if __name__ == "__main__":
    main()

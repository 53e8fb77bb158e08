"""Seeded synthetic inputs with the shapes and distributions of the
workloads the SmoothQuant pages describe (OPT / Llama-2 linears whose
activations carry a few channels about 100x larger than the rest).

This module only draws random numbers: it holds none of the method's
arithmetic, and both the CUDA path and the CPU oracle consume its output.

The pages calibrate on WikiText-2 samples and evaluate real OPT / Llama-2
checkpoints; neither is available here, so these draws stand in for them:
  - activations: rows of N(0,1) (or Student-t with 3 degrees of freedom, or
    SiLU(a)*b of two N(0,1) draws for a down-projection input) with a seeded
    set of outlier channels multiplied by a fixed per-channel factor;
  - weights: N(0, 0.02^2), no outliers.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


# ---------------------------------------------------------------------------
# layer shapes (K = in features, N = out features)
# ---------------------------------------------------------------------------
OPT_6_7B = [("qkv", 4096, 12288), ("out", 4096, 4096), ("fc1", 4096, 16384), ("fc2", 16384, 4096)]
LLAMA2_7B = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
             ("gate", 4096, 11008), ("up", 4096, 11008), ("down", 11008, 4096)]
LLAMA2_70B = [("q", 8192, 8192), ("k", 8192, 1024), ("v", 8192, 1024), ("o", 8192, 8192),
              ("gate", 8192, 28672), ("up", 8192, 28672), ("down", 28672, 8192)]


@dataclass(frozen=True)
class Outliers:
    """Outlier channels and their fixed multipliers."""
    idx: torch.Tensor   # int64 [n]
    mult: torch.Tensor  # float32 [n]


def gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def outliers(K: int, frac: float | None = None, count: int | None = None, mult: float | tuple = 100.0,
             seed: int = 0) -> Outliers:
    """The first round(frac*K) (or `count`) channels of a seeded permutation;
    mult is a constant or a (lo, hi) range drawn uniformly per channel."""
    g = gen(seed)
    n = count if count is not None else int(round(frac * K))
    idx = torch.randperm(K, generator=g)[:n]
    if isinstance(mult, tuple):
        m = torch.rand(n, generator=g) * (mult[1] - mult[0]) + mult[0]
    else:
        m = torch.full((n,), float(mult))
    return Outliers(idx=idx, mult=m.to(torch.float32))


def activations(M: int, K: int, out: Outliers, seed: int, dtype=torch.float32, kind: str = "normal",
                device="cpu") -> torch.Tensor:
    """[M, K] activations; `kind` is 'normal', 'student_t3' or 'silu_mul'."""
    g = gen(seed, device)
    if kind == "normal":
        x = torch.randn(M, K, generator=g, device=device)
    elif kind == "student_t3":
        z = torch.randn(M, K, generator=g, device=device)
        chi2 = torch.zeros(M, K, device=device)
        for _ in range(3):
            chi2 += torch.randn(M, K, generator=g, device=device) ** 2
        x = z / torch.sqrt(chi2 / 3.0)
    elif kind == "silu_mul":
        a = torch.randn(M, K, generator=g, device=device)
        b = torch.randn(M, K, generator=g, device=device)
        x = torch.nn.functional.silu(a) * b
    else:
        raise ValueError(kind)
    if out.idx.numel():
        x[:, out.idx.to(device)] *= out.mult.to(device)
    return x.to(dtype)


def weights(K: int, N: int, seed: int, dtype=torch.float32, layout: str = "nk", std: float = 0.02,
            device="cpu") -> torch.Tensor:
    """N(0, std^2) weights, [N, K] ('nk', nn.Linear) or [K, N] ('kn')."""
    g = gen(seed, device)
    w = torch.randn(N, K, generator=g, device=device) * std
    if layout == "kn":
        w = w.t().contiguous()
    return w.to(dtype)


# ---------------------------------------------------------------------------
# the workloads
# ---------------------------------------------------------------------------

def single_linear_small(seed: int = 1000):
    """Single smoothed linear, alpha 0.5: X fp32 [16, 256] N(0,1) with 4
    outlier channels x100; W fp32 [K=256, N=256] N(0, 0.02); calibration
    stream of 64 tokens from the same distribution; fp32 output."""
    K, N, M = 256, 256, 16
    o = outliers(K, count=4, mult=100.0, seed=seed)
    return dict(
        name="single_linear_16x256x256_f32",
        calib=activations(64, K, o, seed + 1),
        x=activations(M, K, o, seed + 2),
        w=weights(K, N, seed + 3, layout="kn"),
        layout="kn", alpha=0.5, out_dtype=torch.float32, K=K, N=N, M=M,
    )


def opt67b_layer(layer: int, M: int = 2048, calib_tokens: int = 128 * 512, seed: int = 2000, device="cpu",
                 with_calib: bool = True):
    """One OPT-6.7B-shaped linear in fp16: weights N(0, 0.02) as [N, K]
    (nn.Linear layout), activations N(0,1) with 1% of channels scaled by a
    per-channel factor drawn from U(20, 120); M = 2048 prefill tokens;
    calibration 128 x 512 tokens; alpha 0.5."""
    name, K, N = OPT_6_7B[layer]
    s = seed + 10 * layer
    o = outliers(K, frac=0.01, mult=(20.0, 120.0), seed=s)
    d = dict(name=f"opt6.7b_{name}_{K}x{N}", K=K, N=N, M=M, layout="nk", alpha=0.5, out_dtype=torch.float16,
             outliers=o,
             x=activations(M, K, o, s + 1, torch.float16, device=device),
             w=weights(K, N, s + 2, torch.float16, "nk", device=device))
    if with_calib:
        d["calib"] = activations(calib_tokens, K, o, s + 3, torch.float16, device=device)
    return d


def llama_layer(shapes, layer: int, M: int, alpha: float = 0.5, seed: int = 3000, calib_tokens: int = 4096,
                device="cpu"):
    """A Llama-2 decoder linear in bf16: activations N(0,1) with 0.5% fixed
    outlier channels x100 (the down projection's input is SiLU(a)*b of two
    N(0,1) draws, with the same outlier scaling); weights N(0, 0.02) [N, K]."""
    name, K, N = shapes[layer]
    s = seed + 10 * layer
    o = outliers(K, frac=0.005, mult=100.0, seed=s)
    kind = "silu_mul" if name == "down" else "normal"
    return dict(name=f"llama_{name}_{K}x{N}_M{M}", K=K, N=N, M=M, layout="nk", alpha=alpha,
                out_dtype=torch.bfloat16,
                calib=activations(calib_tokens, K, o, s + 3, torch.bfloat16, kind, device=device),
                x=activations(M, K, o, s + 1, torch.bfloat16, kind, device=device),
                w=weights(K, N, s + 2, torch.bfloat16, "nk", device=device))


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def chunks(T: int, size: int):
    """(start, stop) pairs covering [0, T) in pieces of `size`."""
    return [(i, min(T, i + size)) for i in range(0, T, size)]


__all__ = ["OPT_6_7B", "LLAMA2_7B", "LLAMA2_70B", "Outliers", "gen", "outliers", "activations", "weights",
           "single_linear_small", "opt67b_layer", "llama_layer", "ceil_div", "chunks"]

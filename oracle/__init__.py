"""CPU oracle for the SmoothQuant W8A8 smoothed linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference legs of ``bench.py`` may import this package.
It shares no code with the CUDA library: the arithmetic lives in
``sq_oracle.c`` (plain single-threaded C, fp32, round-to-nearest-even, no
FMA contraction); this module only compiles it with gcc and marshals numpy
arrays into it.

Method source: "SmoothQuant (activation smoothing quantization)", jisaku.com
glossary (2023), sections "The mathematics of the smoothing transformation"
(Y = (X diag(s)^-1)(diag(s) W)) and "Hyper-parameter alpha"
(s_j = max|X_j|^alpha / max|W_j|^(1-alpha)).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libsq_oracle.so")

# -O2 without fast-math and without FMA contraction: every fp32 operation is
# one IEEE-rounded operation in source order.
CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared", "-std=gnu11"]

LAYOUT_KN = 0
LAYOUT_NK = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile sq_oracle.c into _build/libsq_oracle.so (gcc)."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        f32p = ctypes.POINTER(ctypes.c_float)
        i8p = ctypes.POINTER(ctypes.c_int8)
        i32p = ctypes.POINTER(ctypes.c_int32)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        f64p = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.c_int64
        sig = {
            "or_quantize_value": ([ctypes.c_float, ctypes.c_float], ctypes.c_int8),
            "or_calib_absmax": ([f32p, i64, i64, f32p], None),
            "or_weight_absmax": ([f32p, ctypes.c_int, i64, i64, f32p], None),
            "or_smooth_factor": ([f32p, f32p, i64, ctypes.c_float, f32p, f32p], None),
            "or_smooth_weight": ([f32p, ctypes.c_int, i64, i64, f32p, f32p], None),
            "or_smooth_quant_weight": ([f32p, ctypes.c_int, i64, i64, f32p, i8p, f32p], None),
            "or_smooth_act": ([f32p, i64, i64, f32p, f32p], None),
            "or_quant_act": ([f32p, i64, i64, f32p, i8p, f32p], None),
            "or_gemm_i8": ([i8p, i8p, i64, i64, i64, i32p], None),
            "or_dequant": ([i32p, f32p, f32p, i64, i64, f32p], None),
            "or_round_bf16": ([f32p, i64, u16p], None),
            "or_round_f16": ([f32p, i64, u16p], None),
            "or_fold_norm_weight": ([f32p, f32p, i64, f32p], None),
            "or_rmsnorm_quant_act": ([f32p, i64, i64, f32p, ctypes.c_float, i8p, f32p], None),
            "or_rmsnorm_factor": ([f32p, i64, i64, ctypes.c_float, f32p], None),
            "or_layernorm_quant_act": ([f32p, i64, i64, f32p, f32p, ctypes.c_float, i8p, f32p], None),
            "or_layernorm_stats": ([f32p, i64, i64, ctypes.c_float, f32p, f32p], None),
            "or_layernorm_values": ([f32p, i64, i64, f32p, f32p, ctypes.c_float, f32p], None),
            "or_static_act_scale": ([f32p, f32p, i64], ctypes.c_float),
            "or_quant_act_static": ([f32p, i64, i64, f32p, ctypes.c_float, i8p, f32p], None),
            "or_e4m3_decode": ([ctypes.c_uint8], ctypes.c_float),
            "or_e4m3_encode": ([ctypes.c_float], ctypes.c_uint8),
            "or_smooth_quant_weight_e4m3": ([f32p, ctypes.c_int, i64, i64, f32p, u8p, f32p], None),
            "or_quant_act_e4m3": ([f32p, i64, i64, f32p, u8p, f32p], None),
            "or_gemm_e4m3": ([u8p, u8p, i64, i64, i64, f64p], None),
            "or_dequant_f32acc": ([f32p, f32p, f32p, i64, i64, f32p], None),
            "or_butterfly_rotate": ([f32p, i64, i64, f32p, f32p], None),
            "or_quant_act_rotated": ([f32p, i64, i64, f32p, i64, f32p, f32p, f32p, i8p, f32p], None),
            "or_smooth_quant_weight_rotated": ([f32p, ctypes.c_int, i64, i64, f32p, i64, f32p, f32p, f32p, i8p,
                                                f32p], None),
        }
        for name, (args, res) in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib


def _f32(a) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    return a


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


# ---------------------------------------------------------------------------
# numpy-facing wrappers, one per oracle step
# ---------------------------------------------------------------------------

def quantize_value(v: float, delta: float) -> int:
    """clamp(rne(v / delta), -127, 127) in fp32 (IEEE division)."""
    return int(_load().or_quantize_value(ctypes.c_float(v), ctypes.c_float(delta)))


def calib_absmax(x, amax=None) -> np.ndarray:
    """Running per-channel max|X_j| over the tokens (rows) of x [T, K]."""
    x = _f32(x)
    T, K = x.shape
    out = np.zeros(K, np.float32) if amax is None else _f32(amax).copy()
    _load().or_calib_absmax(_ptr(x, ctypes.c_float), T, K, _ptr(out, ctypes.c_float))
    return out


def weight_absmax(w, layout: int) -> np.ndarray:
    """w_j = max_n |W_jn| for W given as [K,N] (LAYOUT_KN) or [N,K] (LAYOUT_NK)."""
    w = _f32(w)
    K, N = _kn(w, layout)
    out = np.zeros(K, np.float32)
    _load().or_weight_absmax(_ptr(w, ctypes.c_float), layout, K, N, _ptr(out, ctypes.c_float))
    return out


def smooth_factor(amax, wmax, alpha: float):
    """(s, inv_s) from the per-channel maxima and alpha."""
    amax = _f32(amax)
    wmax = _f32(wmax)
    K = amax.shape[0]
    s = np.zeros(K, np.float32)
    inv = np.zeros(K, np.float32)
    _load().or_smooth_factor(_ptr(amax, ctypes.c_float), _ptr(wmax, ctypes.c_float), K,
                             ctypes.c_float(alpha), _ptr(s, ctypes.c_float), _ptr(inv, ctypes.c_float))
    return s, inv


def smooth_weight(w, layout: int, s) -> np.ndarray:
    """W~ = diag(s) W, returned in W's own layout."""
    w = _f32(w)
    s = _f32(s)
    K, N = _kn(w, layout)
    out = np.zeros_like(w)
    _load().or_smooth_weight(_ptr(w, ctypes.c_float), layout, K, N, _ptr(s, ctypes.c_float),
                             _ptr(out, ctypes.c_float))
    return out


def smooth_quant_weight(w, layout: int, s):
    """(Wq [N,K] int8, dw [N] fp32) from W and s."""
    w = _f32(w)
    s = _f32(s)
    K, N = _kn(w, layout)
    wq = np.zeros((N, K), np.int8)
    dw = np.zeros(N, np.float32)
    _load().or_smooth_quant_weight(_ptr(w, ctypes.c_float), layout, K, N, _ptr(s, ctypes.c_float),
                                   _ptr(wq, ctypes.c_int8), _ptr(dw, ctypes.c_float))
    return wq, dw


def smooth_act(x, inv_s) -> np.ndarray:
    """X~ = X diag(s)^-1 = X * inv_s (per column)."""
    x = _f32(x)
    inv_s = _f32(inv_s)
    M, K = x.shape
    out = np.zeros_like(x)
    _load().or_smooth_act(_ptr(x, ctypes.c_float), M, K, _ptr(inv_s, ctypes.c_float),
                          _ptr(out, ctypes.c_float))
    return out


def quant_act(x, inv_s):
    """(Xq [M,K] int8, dx [M] fp32): smoothing then per-token quantization."""
    x = _f32(x)
    inv_s = _f32(inv_s)
    M, K = x.shape
    xq = np.zeros((M, K), np.int8)
    dx = np.zeros(M, np.float32)
    _load().or_quant_act(_ptr(x, ctypes.c_float), M, K, _ptr(inv_s, ctypes.c_float),
                         _ptr(xq, ctypes.c_int8), _ptr(dx, ctypes.c_float))
    return xq, dx


def gemm_i8(xq, wq) -> np.ndarray:
    """acc [M,N] int32 = Xq [M,K] . Wq[N,K]^T."""
    xq = np.ascontiguousarray(np.asarray(xq, dtype=np.int8))
    wq = np.ascontiguousarray(np.asarray(wq, dtype=np.int8))
    M, K = xq.shape
    N, K2 = wq.shape
    assert K == K2
    acc = np.zeros((M, N), np.int32)
    _load().or_gemm_i8(_ptr(xq, ctypes.c_int8), _ptr(wq, ctypes.c_int8), M, N, K, _ptr(acc, ctypes.c_int32))
    return acc


def dequant(acc, dx, dw) -> np.ndarray:
    """y [M,N] fp32 = ((float)acc * dx_t) * dw_n."""
    acc = np.ascontiguousarray(np.asarray(acc, dtype=np.int32))
    dx = _f32(dx)
    dw = _f32(dw)
    M, N = acc.shape
    y = np.zeros((M, N), np.float32)
    _load().or_dequant(_ptr(acc, ctypes.c_int32), _ptr(dx, ctypes.c_float), _ptr(dw, ctypes.c_float),
                       M, N, _ptr(y, ctypes.c_float))
    return y


def round_to(y, dtype: str) -> np.ndarray:
    """Round fp32 y to 'bf16' / 'f16' (returned as raw uint16 bit patterns) or keep 'f32'."""
    y = _f32(y)
    if dtype == "f32":
        return y.copy()
    out = np.zeros(y.shape, np.uint16)
    fn = _load().or_round_bf16 if dtype == "bf16" else _load().or_round_f16
    if dtype not in ("bf16", "f16"):
        raise ValueError(dtype)
    fn(_ptr(y, ctypes.c_float), y.size, _ptr(out, ctypes.c_uint16))
    return out


def fold_norm_weight(gamma, inv_s) -> np.ndarray:
    """gs_j = gamma_j * inv_s_j: diag(s)^-1 folded into the norm's weight."""
    gamma = _f32(gamma)
    inv_s = _f32(inv_s)
    gs = np.zeros(gamma.shape[0], np.float32)
    _load().or_fold_norm_weight(_ptr(gamma, ctypes.c_float), _ptr(inv_s, ctypes.c_float), gamma.shape[0],
                                _ptr(gs, ctypes.c_float))
    return gs


def rmsnorm_quant_act(x, gs, eps: float):
    """(Xq, dx): RMSNorm (epsilon eps) with the folded weight gs, then
    per-token quantization."""
    x = _f32(x)
    gs = _f32(gs)
    M, K = x.shape
    xq = np.zeros((M, K), np.int8)
    dx = np.zeros(M, np.float32)
    _load().or_rmsnorm_quant_act(_ptr(x, ctypes.c_float), M, K, _ptr(gs, ctypes.c_float), ctypes.c_float(eps),
                                 _ptr(xq, ctypes.c_int8), _ptr(dx, ctypes.c_float))
    return xq, dx


def rmsnorm_factor(x, eps: float) -> np.ndarray:
    """Per-token r_t = 1 / sqrt(mean_j x_tj^2 + eps), rounded once to fp32."""
    x = _f32(x)
    M, K = x.shape
    r = np.zeros(M, np.float32)
    _load().or_rmsnorm_factor(_ptr(x, ctypes.c_float), M, K, ctypes.c_float(eps), _ptr(r, ctypes.c_float))
    return r


def layernorm_quant_act(x, gs, bs, eps: float):
    """(Xq, dx): LayerNorm (epsilon eps) with the folded weight gs and bias
    bs (None: no bias), then per-token quantization."""
    x = _f32(x)
    gs = _f32(gs)
    M, K = x.shape
    xq = np.zeros((M, K), np.int8)
    dx = np.zeros(M, np.float32)
    bp = None if bs is None else _f32(bs)
    _load().or_layernorm_quant_act(_ptr(x, ctypes.c_float), M, K, _ptr(gs, ctypes.c_float),
                                   None if bp is None else _ptr(bp, ctypes.c_float), ctypes.c_float(eps),
                                   _ptr(xq, ctypes.c_int8), _ptr(dx, ctypes.c_float))
    return xq, dx


def layernorm_stats(x, eps: float):
    """Per-token (mu_t, r_t): the mean rounded once to fp32, and
    1 / sqrt(var_t + eps) rounded once to fp32."""
    x = _f32(x)
    M, K = x.shape
    mu = np.zeros(M, np.float32)
    r = np.zeros(M, np.float32)
    _load().or_layernorm_stats(_ptr(x, ctypes.c_float), M, K, ctypes.c_float(eps), _ptr(mu, ctypes.c_float),
                               _ptr(r, ctypes.c_float))
    return mu, r


def layernorm_values(x, gs, bs, eps: float) -> np.ndarray:
    """The folded LayerNorm values v [M,K] that layernorm_quant_act quantizes."""
    x = _f32(x)
    gs = _f32(gs)
    M, K = x.shape
    v = np.zeros((M, K), np.float32)
    bp = None if bs is None else _f32(bs)
    _load().or_layernorm_values(_ptr(x, ctypes.c_float), M, K, _ptr(gs, ctypes.c_float),
                                None if bp is None else _ptr(bp, ctypes.c_float), ctypes.c_float(eps),
                                _ptr(v, ctypes.c_float))
    return v


def static_act_scale(amax, inv_s) -> float:
    """Per-tensor scale max_j(a_j * inv_s_j) / 127 from calibration maxima."""
    amax = _f32(amax)
    inv_s = _f32(inv_s)
    return float(_load().or_static_act_scale(_ptr(amax, ctypes.c_float), _ptr(inv_s, ctypes.c_float),
                                             amax.shape[0]))


def quant_act_static(x, inv_s, delta: float):
    """(Xq, dx): smoothing then quantization with one fixed scale delta."""
    x = _f32(x)
    inv_s = _f32(inv_s)
    M, K = x.shape
    xq = np.zeros((M, K), np.int8)
    dx = np.zeros(M, np.float32)
    _load().or_quant_act_static(_ptr(x, ctypes.c_float), M, K, _ptr(inv_s, ctypes.c_float), ctypes.c_float(delta),
                                _ptr(xq, ctypes.c_int8), _ptr(dx, ctypes.c_float))
    return xq, dx


# ---------------------------------------------------------------------------
# FP8 (E4M3) variant
# ---------------------------------------------------------------------------

def e4m3_decode(codes) -> np.ndarray:
    """Exact float value of each E4M3 code (uint8 array)."""
    c = np.asarray(codes, dtype=np.uint8)
    f = _load().or_e4m3_decode
    return np.array([f(int(v)) for v in c.ravel()], np.float32).reshape(c.shape)


def e4m3_encode(values) -> np.ndarray:
    """Nearest E4M3 code of each fp32 value (ties to even, +-448 beyond)."""
    v = _f32(values)
    f = _load().or_e4m3_encode
    return np.array([f(float(x)) for x in v.ravel()], np.uint8).reshape(v.shape)


def smooth_quant_weight_e4m3(w, layout: int, s):
    """(Wq [N, K] uint8 E4M3 codes, dw [N]) of W~ = diag(s) W, per output channel."""
    w = _f32(w)
    s = _f32(s)
    K, N = _kn(w, layout)
    wq = np.zeros((N, K), np.uint8)
    dw = np.zeros(N, np.float32)
    _load().or_smooth_quant_weight_e4m3(_ptr(w, ctypes.c_float), layout, K, N, _ptr(s, ctypes.c_float),
                                        _ptr(wq, ctypes.c_uint8), _ptr(dw, ctypes.c_float))
    return wq, dw


def quant_act_e4m3(x, inv_s):
    """(Xq [M, K] uint8 E4M3 codes, dx [M]) of X~ = X diag(s)^-1, per token."""
    x = _f32(x)
    inv_s = _f32(inv_s)
    M, K = x.shape
    xq = np.zeros((M, K), np.uint8)
    dx = np.zeros(M, np.float32)
    _load().or_quant_act_e4m3(_ptr(x, ctypes.c_float), M, K, _ptr(inv_s, ctypes.c_float),
                              _ptr(xq, ctypes.c_uint8), _ptr(dx, ctypes.c_float))
    return xq, dx


def gemm_e4m3(xq, wq) -> np.ndarray:
    """Exact acc[M, N] = sum_j e4m3(xq[t, j]) e4m3(wq[n, j]) in float64."""
    xq = np.ascontiguousarray(xq, dtype=np.uint8)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    M, K = xq.shape
    N = wq.shape[0]
    acc = np.zeros((M, N), np.float64)
    _load().or_gemm_e4m3(_ptr(xq, ctypes.c_uint8), _ptr(wq, ctypes.c_uint8), M, N, K,
                         _ptr(acc, ctypes.c_double))
    return acc


def dequant_f32acc(acc, dx, dw) -> np.ndarray:
    """y = ((float)acc * dx_t) * dw_n for an fp32 accumulator."""
    acc = _f32(acc)
    dx = _f32(dx)
    dw = _f32(dw)
    M, N = acc.shape
    y = np.zeros((M, N), np.float32)
    _load().or_dequant_f32acc(_ptr(acc, ctypes.c_float), _ptr(dx, ctypes.c_float), _ptr(dw, ctypes.c_float), M, N,
                              _ptr(y, ctypes.c_float))
    return y


# ---------------------------------------------------------------------------
# butterfly rotation (Givens rotations in an FFT butterfly, per n-block)
# ---------------------------------------------------------------------------

def _angles(n: int, c, s):
    L = n.bit_length() - 1
    if n < 2 or (1 << L) != n:
        raise ValueError("n must be a power of two >= 2")
    c = _f32(c).reshape(L, n // 2)
    s = _f32(s).reshape(L, n // 2)
    return np.ascontiguousarray(c), np.ascontiguousarray(s)


def butterfly_rotate(v, n: int, c, s) -> np.ndarray:
    """Every row of v [rows, K] rotated block by block (K % n == 0) by the
    butterfly with cos/sin tables c, s [log2 n, n/2]."""
    v = _f32(v).copy()
    c, s = _angles(n, c, s)
    rows, K = v.shape
    for r in range(rows):
        row = np.ascontiguousarray(v[r])
        _load().or_butterfly_rotate(_ptr(row, ctypes.c_float), K, n, _ptr(c, ctypes.c_float), _ptr(s, ctypes.c_float))
        v[r] = row
    return v


def quant_act_rotated(x, inv_s, n: int, c, s):
    """(Xq, dx): per-token INT8 of the rotated smoothed activations R(x * inv_s)."""
    x = _f32(x)
    inv_s = _f32(inv_s)
    c, s = _angles(n, c, s)
    M, K = x.shape
    xq = np.zeros((M, K), np.int8)
    dx = np.zeros(M, np.float32)
    work = np.zeros(K, np.float32)
    _load().or_quant_act_rotated(_ptr(x, ctypes.c_float), M, K, _ptr(inv_s, ctypes.c_float), n,
                                 _ptr(c, ctypes.c_float), _ptr(s, ctypes.c_float), _ptr(work, ctypes.c_float),
                                 _ptr(xq, ctypes.c_int8), _ptr(dx, ctypes.c_float))
    return xq, dx


def smooth_quant_weight_rotated(w, layout: int, smooth, n: int, c, s):
    """(Wq [N, K], dw [N]) of the rotated smoothed weights R(s * w_n)."""
    w = _f32(w)
    smooth = _f32(smooth)
    c, s = _angles(n, c, s)
    K, N = _kn(w, layout)
    wq = np.zeros((N, K), np.int8)
    dw = np.zeros(N, np.float32)
    work = np.zeros(K, np.float32)
    _load().or_smooth_quant_weight_rotated(_ptr(w, ctypes.c_float), layout, K, N, _ptr(smooth, ctypes.c_float), n,
                                           _ptr(c, ctypes.c_float), _ptr(s, ctypes.c_float),
                                           _ptr(work, ctypes.c_float), _ptr(wq, ctypes.c_int8),
                                           _ptr(dw, ctypes.c_float))
    return wq, dw


def linear(x, inv_s, wq, dw, out_dtype: str = "f32"):
    """The runtime smoothed linear: quant_act -> gemm_i8 -> dequant -> round."""
    xq, dx = quant_act(x, inv_s)
    acc = gemm_i8(xq, wq)
    y = dequant(acc, dx, dw)
    return round_to(y, out_dtype), acc, xq, dx


def pipeline(calib_chunks, w, layout: int, alpha: float, x, out_dtype: str = "f32"):
    """Whole path in the usage order: calibrate -> smooth+quantize W -> linear."""
    K = _kn(_f32(w), layout)[0]
    amax = np.zeros(K, np.float32)
    for c in calib_chunks:
        amax = calib_absmax(c, amax)
    wmax = weight_absmax(w, layout)
    s, inv_s = smooth_factor(amax, wmax, alpha)
    wq, dw = smooth_quant_weight(w, layout, s)
    y, acc, xq, dx = linear(x, inv_s, wq, dw, out_dtype)
    return dict(amax=amax, wmax=wmax, s=s, inv_s=inv_s, wq=wq, dw=dw, xq=xq, dx=dx, acc=acc, y=y)


def _kn(w: np.ndarray, layout: int):
    if layout == LAYOUT_KN:
        return w.shape[0], w.shape[1]
    if layout == LAYOUT_NK:
        return w.shape[1], w.shape[0]
    raise ValueError(f"layout {layout}")

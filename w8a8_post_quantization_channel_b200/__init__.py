"""SmoothQuant W8A8 smoothed linear layer on B200 (sm_100a).

Thin Python binding over the C ABI of ``libsq.so`` (declared in
``include/sq.h``).  Each function has the C call's name and only marshals
arguments: tensors become device pointers, sizes and leading dimensions;
torch provides memory and the current CUDA stream.  Every step of the path
runs in the library's kernels; there is no fallback: if the library cannot
be loaded, every call raises.

Method ("SmoothQuant (activation smoothing quantization)", jisaku.com
glossary): Y = (X diag(s)^-1)(diag(s) W) with
s_j = max|X_j|^alpha / max|W_j|^(1-alpha), both operands quantized to INT8
and multiplied on INT8 tensor cores.  Usage order, as on the page:

    amax = torch.zeros(K, device="cuda")
    for chunk in calibration_stream:             # get_act_scales
        sq_calib_absmax(chunk, amax)
    wq, w_scale, s, inv_s = sq_smooth_quant_weight(w, SQ_W_NK, amax, 0.5)
    xq, x_scale = sq_quant_act(x, inv_s)         # smooth_lm + quantize
    y = sq_w8a8_linear(xq, x_scale, wq, w_scale, out_dtype=torch.bfloat16)
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

__all__ = [
    "SQ_OK", "SQ_ERR_INVALID_ARG", "SQ_ERR_UNSUPPORTED", "SQ_ERR_CUDA", "SQ_ERR_TIMEOUT",
    "SQ_F32", "SQ_F16", "SQ_BF16", "SQ_W_KN", "SQ_W_NK", "SqError",
    "lib", "library_path", "header_functions",
    "sq_calib_absmax", "sq_smooth_quant_weight", "sq_quant_act", "sq_w8a8_linear",
    "sq_w8a8_linear_workspace_size", "sq_w8a8_accumulate", "sq_check_device_error", "sq_status_string",
    "sq_w8a8_linear_decode_noalloc", "SQ_DECODE_STATIC_SCRATCH_BYTES", "sq_decode_static_scratch_bytes",
    "sq_selftest_wait_timeout",
    "sq_fold_smooth_into_norm", "sq_rmsnorm_quant_act", "sq_layernorm_quant_act", "sq_static_act_scale",
    "sq_quant_act_static",
    "sq_smooth_quant_weight_e4m3", "sq_quant_act_e4m3", "sq_w8a8_linear_e4m3", "sq_w8a8_accumulate_e4m3",
    "sq_w8a8_linear_scatter", "sq_quant_act_rotated", "sq_smooth_quant_weight_rotated",
]

SQ_OK, SQ_ERR_INVALID_ARG, SQ_ERR_UNSUPPORTED, SQ_ERR_CUDA, SQ_ERR_TIMEOUT = 0, 1, 2, 3, 4
SQ_F32, SQ_F16, SQ_BF16 = 0, 1, 2
SQ_W_KN, SQ_W_NK = 0, 1

_PKG = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_PKG)
_HEADER = os.path.join(_ROOT, "include", "sq.h")
_LIB_PATH = os.path.join(_PKG, "libsq.so")
_DT = {torch.float32: SQ_F32, torch.float16: SQ_F16, torch.bfloat16: SQ_BF16}
_lib = None


class SqError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {sq_status_string(status)} ({status})")
        self.status = status


def library_path() -> str:
    """Path of the in-tree libsq.so this binding loads."""
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Loads libsq.so (building it in-tree first when it is missing or stale)."""
    global _lib
    if _lib is None:
        from . import build as _build
        try:
            path = _build.build()
        except Exception as e:  # no nvcc: only an existing library will do
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(f"libsq.so is missing and cannot be built: {e}") from e
            path = _LIB_PATH
        L = ctypes.CDLL(path)
        vp, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        sigs = {
            "sq_calib_absmax": [vp, i32, i64, i64, i64, vp, vp],
            "sq_smooth_quant_weight": [vp, i32, i32, i64, i64, i64, vp, f32, vp, vp, vp, vp, vp],
            "sq_quant_act": [vp, i32, i64, i64, i64, vp, vp, vp, vp],
            "sq_w8a8_linear": [vp, vp, vp, vp, i64, i64, i64, vp, i32, i64, vp, sz, vp],
            "sq_w8a8_accumulate": [vp, vp, i64, i64, i64, vp, i64, vp, sz, vp],
            "sq_check_device_error": [vp],
            "sq_w8a8_linear_decode_noalloc": [vp, vp, vp, vp, i64, i64, i64, vp, i32, i64, vp],
            "sq_selftest_wait_timeout": [i32, vp],
            "sq_fold_smooth_into_norm": [vp, vp, i64, vp, vp],
            "sq_rmsnorm_quant_act": [vp, i32, i64, i64, i64, vp, f32, vp, vp, vp],
            "sq_layernorm_quant_act": [vp, i32, i64, i64, i64, vp, vp, f32, vp, vp, vp],
            "sq_static_act_scale": [vp, vp, i64, vp, vp],
            "sq_quant_act_static": [vp, i32, i64, i64, i64, vp, vp, vp, vp, vp],
            "sq_smooth_quant_weight_e4m3": [vp, i32, i32, i64, i64, i64, vp, f32, vp, vp, vp, vp, vp],
            "sq_quant_act_e4m3": [vp, i32, i64, i64, i64, vp, vp, vp, vp],
            "sq_w8a8_linear_e4m3": [vp, vp, vp, vp, i64, i64, i64, vp, i32, i64, vp, sz, vp],
            "sq_w8a8_accumulate_e4m3": [vp, vp, i64, i64, i64, vp, i64, vp, sz, vp],
            "sq_w8a8_linear_scatter": [vp, vp, vp, vp, i64, i64, i64, vp, i32, i32, i64, vp, sz, vp],
            "sq_quant_act_rotated": [vp, i32, i64, i64, i64, vp, i64, vp, vp, vp, vp],
            "sq_smooth_quant_weight_rotated": [vp, i32, i64, i64, i64, vp, f32, i64, vp, vp, vp, vp, vp, vp],
        }
        for name, args in sigs.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.sq_decode_static_scratch_bytes.argtypes = []
        L.sq_decode_static_scratch_bytes.restype = sz
        L.sq_w8a8_linear_workspace_size.argtypes = [i64, i64, i64]
        L.sq_w8a8_linear_workspace_size.restype = sz
        L.sq_status_string.argtypes = [ctypes.c_int]
        L.sq_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/sq.h declares."""
    with open(_HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(sq_\w+)\s*\(", text, flags=re.M)


def sq_status_string(status: int) -> str:
    """The library's description of a status code."""
    return lib().sq_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != SQ_OK:
        raise SqError(status, what)


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


# Zeroed workspaces of the linear entry points, one per (device, stream).
# Every call leaves its workspace zero again and calls on one stream run in
# order, so one buffer serves them all; it grows to the largest need seen.
_WORKSPACES: dict = {}


def _workspace(need: int, device, stream):
    if need == 0:
        return None
    s = stream if stream is not None else torch.cuda.current_stream(device)
    key = (torch.device(device).index, s.cuda_stream)
    w = _WORKSPACES.get(key)
    if w is None or w.numel() < need:
        with torch.cuda.stream(s):  # allocated on the stream that uses it
            w = torch.zeros(need, dtype=torch.uint8, device=device)
        _WORKSPACES[key] = w
    return w


def _rowmajor(t: torch.Tensor, name: str) -> None:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D tensor with unit column stride")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")


def _dtype(t: torch.Tensor, name: str) -> int:
    if t.dtype not in _DT:
        raise ValueError(f"{name}: dtype {t.dtype} not supported (float32/float16/bfloat16)")
    return _DT[t.dtype]


def sq_calib_absmax(x: torch.Tensor, amax: torch.Tensor, stream=None) -> torch.Tensor:
    """amax[K] (fp32, in-out) <- max(amax, max over tokens of |x|); x is [T, K]."""
    _rowmajor(x, "x")
    _check(lib().sq_calib_absmax(_ptr(x), _dtype(x, "x"), x.shape[0], x.shape[1], x.stride(0), _ptr(amax),
                                 _stream(stream)), "sq_calib_absmax")
    return amax


def sq_smooth_quant_weight(w: torch.Tensor, layout: int, amax: torch.Tensor, alpha: float = 0.5,
                           wq=None, w_scale=None, smooth=None, inv_smooth=None, stream=None):
    """(wq [N,K] int8, w_scale [N], s [K], inv_s [K]) from W ([K,N] for SQ_W_KN, [N,K] for SQ_W_NK)."""
    _rowmajor(w, "w")
    K, N = (w.shape[0], w.shape[1]) if layout == SQ_W_KN else (w.shape[1], w.shape[0])
    dev = w.device
    wq = torch.empty((N, K), dtype=torch.int8, device=dev) if wq is None else wq
    w_scale = torch.empty(N, dtype=torch.float32, device=dev) if w_scale is None else w_scale
    smooth = torch.empty(K, dtype=torch.float32, device=dev) if smooth is None else smooth
    inv_smooth = torch.empty(K, dtype=torch.float32, device=dev) if inv_smooth is None else inv_smooth
    _check(lib().sq_smooth_quant_weight(_ptr(w), _dtype(w, "w"), layout, K, N, w.stride(0), _ptr(amax),
                                        ctypes.c_float(alpha), _ptr(wq), _ptr(w_scale), _ptr(smooth),
                                        _ptr(inv_smooth), _stream(stream)), "sq_smooth_quant_weight")
    return wq, w_scale, smooth, inv_smooth


def sq_quant_act(x: torch.Tensor, inv_smooth: torch.Tensor, xq=None, x_scale=None, stream=None):
    """(xq [M,K] int8, x_scale [M]) = per-token INT8 of x * inv_smooth."""
    _rowmajor(x, "x")
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device) if xq is None else xq
    x_scale = torch.empty(M, dtype=torch.float32, device=x.device) if x_scale is None else x_scale
    _check(lib().sq_quant_act(_ptr(x), _dtype(x, "x"), M, K, x.stride(0), _ptr(inv_smooth), _ptr(xq),
                              _ptr(x_scale), _stream(stream)), "sq_quant_act")
    return xq, x_scale


def sq_quant_act_rotated(x: torch.Tensor, inv_smooth: torch.Tensor, n: int, rot_cs: torch.Tensor, xq=None,
                         x_scale=None, stream=None):
    """(xq, x_scale) = per-token INT8 of the butterfly rotation (blocks of n,
    (cos, sin) table rot_cs [log2 n, n/2, 2]) of x * inv_smooth."""
    _rowmajor(x, "x")
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device) if xq is None else xq
    x_scale = torch.empty(M, dtype=torch.float32, device=x.device) if x_scale is None else x_scale
    _check(lib().sq_quant_act_rotated(_ptr(x), _dtype(x, "x"), M, K, x.stride(0), _ptr(inv_smooth), n, _ptr(rot_cs),
                                      _ptr(xq), _ptr(x_scale), _stream(stream)), "sq_quant_act_rotated")
    return xq, x_scale


def sq_smooth_quant_weight_rotated(w: torch.Tensor, amax: torch.Tensor, alpha: float, n: int, rot_cs: torch.Tensor,
                                   wq=None, w_scale=None, smooth=None, inv_smooth=None, stream=None):
    """(wq [N,K] int8, w_scale, s, inv_s) with every output channel's smoothed
    K-vector rotated like the activations; w is [N, K] (nn.Linear layout)."""
    _rowmajor(w, "w")
    N, K = w.shape
    dev = w.device
    wq = torch.empty((N, K), dtype=torch.int8, device=dev) if wq is None else wq
    w_scale = torch.empty(N, dtype=torch.float32, device=dev) if w_scale is None else w_scale
    smooth = torch.empty(K, dtype=torch.float32, device=dev) if smooth is None else smooth
    inv_smooth = torch.empty(K, dtype=torch.float32, device=dev) if inv_smooth is None else inv_smooth
    _check(lib().sq_smooth_quant_weight_rotated(_ptr(w), _dtype(w, "w"), K, N, w.stride(0), _ptr(amax),
                                                ctypes.c_float(alpha), n, _ptr(rot_cs), _ptr(wq), _ptr(w_scale),
                                                _ptr(smooth), _ptr(inv_smooth), _stream(stream)),
           "sq_smooth_quant_weight_rotated")
    return wq, w_scale, smooth, inv_smooth


def sq_fold_smooth_into_norm(gamma: torch.Tensor, inv_smooth: torch.Tensor, gs=None, stream=None) -> torch.Tensor:
    """gs = gamma * inv_smooth (fp32): the smoothing folded into the norm weight."""
    gs = torch.empty_like(gamma) if gs is None else gs
    _check(lib().sq_fold_smooth_into_norm(_ptr(gamma), _ptr(inv_smooth), gamma.numel(), _ptr(gs), _stream(stream)),
           "sq_fold_smooth_into_norm")
    return gs


def sq_rmsnorm_quant_act(x: torch.Tensor, gs: torch.Tensor, eps: float, xq=None, x_scale=None, stream=None):
    """(xq, x_scale) = per-token INT8 of RMSNorm(x; eps) with the folded weight gs."""
    _rowmajor(x, "x")
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device) if xq is None else xq
    x_scale = torch.empty(M, dtype=torch.float32, device=x.device) if x_scale is None else x_scale
    _check(lib().sq_rmsnorm_quant_act(_ptr(x), _dtype(x, "x"), M, K, x.stride(0), _ptr(gs), ctypes.c_float(eps),
                                      _ptr(xq), _ptr(x_scale), _stream(stream)), "sq_rmsnorm_quant_act")
    return xq, x_scale


def sq_layernorm_quant_act(x: torch.Tensor, gs: torch.Tensor, bs, eps: float, xq=None, x_scale=None, stream=None):
    """(xq, x_scale) = per-token INT8 of LayerNorm(x; eps) with the folded
    weight gs and bias bs (None: no bias)."""
    _rowmajor(x, "x")
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device) if xq is None else xq
    x_scale = torch.empty(M, dtype=torch.float32, device=x.device) if x_scale is None else x_scale
    _check(lib().sq_layernorm_quant_act(_ptr(x), _dtype(x, "x"), M, K, x.stride(0), _ptr(gs),
                                        None if bs is None else _ptr(bs), ctypes.c_float(eps), _ptr(xq),
                                        _ptr(x_scale), _stream(stream)), "sq_layernorm_quant_act")
    return xq, x_scale


def sq_static_act_scale(amax: torch.Tensor, inv_smooth: torch.Tensor, delta=None, stream=None) -> torch.Tensor:
    """delta (1-element device tensor) = max_j(amax_j * inv_smooth_j) / 127."""
    delta = torch.empty(1, dtype=torch.float32, device=amax.device) if delta is None else delta
    _check(lib().sq_static_act_scale(_ptr(amax), _ptr(inv_smooth), amax.numel(), _ptr(delta), _stream(stream)),
           "sq_static_act_scale")
    return delta


def sq_quant_act_static(x: torch.Tensor, inv_smooth: torch.Tensor, delta: torch.Tensor, xq=None, x_scale=None,
                        stream=None):
    """(xq, x_scale) with one fixed scale *delta (device scalar); saturates."""
    _rowmajor(x, "x")
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device) if xq is None else xq
    x_scale = torch.empty(M, dtype=torch.float32, device=x.device) if x_scale is None else x_scale
    _check(lib().sq_quant_act_static(_ptr(x), _dtype(x, "x"), M, K, x.stride(0), _ptr(inv_smooth), _ptr(delta),
                                     _ptr(xq), _ptr(x_scale), _stream(stream)), "sq_quant_act_static")
    return xq, x_scale


def sq_w8a8_linear_workspace_size(M: int, N: int, K: int) -> int:
    """Workspace bytes sq_w8a8_linear needs for this shape on the current device
    (the stream-K decode shapes; 0 for every other shape)."""
    return int(lib().sq_w8a8_linear_workspace_size(M, N, K))


def sq_w8a8_linear(xq: torch.Tensor, x_scale: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor,
                   out_dtype=torch.bfloat16, y=None, workspace=None, stream=None) -> torch.Tensor:
    """y [M,N] = dequant(xq . wq^T) in out_dtype (float32/float16/bfloat16)."""
    M, K = xq.shape
    N = wq.shape[0]
    y = torch.empty((M, N), dtype=out_dtype, device=xq.device) if y is None else y
    _rowmajor(y, "y")
    need = sq_w8a8_linear_workspace_size(M, N, K)
    if workspace is None:
        workspace = _workspace(need, xq.device, stream)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().sq_w8a8_linear(_ptr(xq), _ptr(x_scale), _ptr(wq), _ptr(w_scale), M, N, K, _ptr(y),
                                _dtype(y, "y"), y.stride(0), _ptr(workspace), wbytes, _stream(stream)),
           "sq_w8a8_linear")
    return y


def sq_w8a8_linear_scatter(xq: torch.Tensor, x_scale: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor,
                           ys, col0: int, workspace=None, stream=None) -> None:
    """Column-parallel linear: this shard's Y[:, col0:col0+N] (wq, w_scale are
    the shard's rows) stored into every full [M, N_total] tensor in ys (this
    rank's Y and peers' copies; all of one dtype and row stride)."""
    M, K = xq.shape
    N = wq.shape[0]
    if not 1 <= len(ys) <= 8:
        raise ValueError("1 to 8 destinations")
    y0 = ys[0]
    for y in ys:
        if y.dim() != 2 or y.stride(1) != 1 or y.dtype != y0.dtype or y.stride(0) != y0.stride(0):
            raise ValueError("destinations must be row-major 2-D tensors of one dtype and row stride")
        if y.shape[0] != M or col0 < 0 or col0 + N > y.shape[1]:
            raise ValueError("shard does not fit the destination")
    esz = y0.element_size()
    ptrs = (ctypes.c_void_p * len(ys))(*[y.data_ptr() + col0 * esz for y in ys])
    need = sq_w8a8_linear_workspace_size(M, N, K)
    if workspace is None:
        workspace = _workspace(need, xq.device, stream)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().sq_w8a8_linear_scatter(_ptr(xq), _ptr(x_scale), _ptr(wq), _ptr(w_scale), M, N, K, ptrs, len(ys),
                                        _dtype(y0, "y"), y0.stride(0), _ptr(workspace), wbytes, _stream(stream)),
           "sq_w8a8_linear_scatter")


def sq_w8a8_accumulate(xq: torch.Tensor, wq: torch.Tensor, acc=None, workspace=None, stream=None) -> torch.Tensor:
    """acc [M,N] int32 = xq . wq^T on the tensor cores (exact)."""
    M, K = xq.shape
    N = wq.shape[0]
    acc = torch.empty((M, N), dtype=torch.int32, device=xq.device) if acc is None else acc
    need = sq_w8a8_linear_workspace_size(M, N, K)
    if workspace is None:
        workspace = _workspace(need, xq.device, stream)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().sq_w8a8_accumulate(_ptr(xq), _ptr(wq), M, N, K, _ptr(acc), acc.stride(0), _ptr(workspace),
                                    wbytes, _stream(stream)), "sq_w8a8_accumulate")
    return acc


# ---------------------------------------------------------------------------
# FP8 (E4M3) variant: codes are uint8 tensors holding E4M3 bit patterns
# ---------------------------------------------------------------------------

def sq_smooth_quant_weight_e4m3(w: torch.Tensor, layout: int, amax: torch.Tensor, alpha: float = 0.5,
                                wq=None, w_scale=None, smooth=None, inv_smooth=None, stream=None):
    """(wq [N,K] uint8 E4M3, w_scale [N] = absmax/448, s [K], inv_s [K])."""
    _rowmajor(w, "w")
    K, N = (w.shape[0], w.shape[1]) if layout == SQ_W_KN else (w.shape[1], w.shape[0])
    dev = w.device
    wq = torch.empty((N, K), dtype=torch.uint8, device=dev) if wq is None else wq
    w_scale = torch.empty(N, dtype=torch.float32, device=dev) if w_scale is None else w_scale
    smooth = torch.empty(K, dtype=torch.float32, device=dev) if smooth is None else smooth
    inv_smooth = torch.empty(K, dtype=torch.float32, device=dev) if inv_smooth is None else inv_smooth
    _check(lib().sq_smooth_quant_weight_e4m3(_ptr(w), _dtype(w, "w"), layout, K, N, w.stride(0), _ptr(amax),
                                             ctypes.c_float(alpha), _ptr(wq), _ptr(w_scale), _ptr(smooth),
                                             _ptr(inv_smooth), _stream(stream)), "sq_smooth_quant_weight_e4m3")
    return wq, w_scale, smooth, inv_smooth


def sq_quant_act_e4m3(x: torch.Tensor, inv_smooth: torch.Tensor, xq=None, x_scale=None, stream=None):
    """(xq [M,K] uint8 E4M3, x_scale [M] = absmax/448) of x * inv_smooth, per token."""
    _rowmajor(x, "x")
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.uint8, device=x.device) if xq is None else xq
    x_scale = torch.empty(M, dtype=torch.float32, device=x.device) if x_scale is None else x_scale
    _check(lib().sq_quant_act_e4m3(_ptr(x), _dtype(x, "x"), M, K, x.stride(0), _ptr(inv_smooth), _ptr(xq),
                                   _ptr(x_scale), _stream(stream)), "sq_quant_act_e4m3")
    return xq, x_scale


def sq_w8a8_linear_e4m3(xq: torch.Tensor, x_scale: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor,
                        out_dtype=torch.bfloat16, y=None, workspace=None, stream=None) -> torch.Tensor:
    """y [M,N] = dequant(xq . wq^T) for E4M3 codes, fp32 accumulation."""
    M, K = xq.shape
    N = wq.shape[0]
    y = torch.empty((M, N), dtype=out_dtype, device=xq.device) if y is None else y
    _rowmajor(y, "y")
    need = sq_w8a8_linear_workspace_size(M, N, K)
    if workspace is None:
        workspace = _workspace(need, xq.device, stream)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().sq_w8a8_linear_e4m3(_ptr(xq), _ptr(x_scale), _ptr(wq), _ptr(w_scale), M, N, K, _ptr(y),
                                     _dtype(y, "y"), y.stride(0), _ptr(workspace), wbytes, _stream(stream)),
           "sq_w8a8_linear_e4m3")
    return y


def sq_w8a8_accumulate_e4m3(xq: torch.Tensor, wq: torch.Tensor, acc=None, workspace=None,
                            stream=None) -> torch.Tensor:
    """acc [M,N] float32 = e4m3(xq) . e4m3(wq)^T on the tensor cores."""
    M, K = xq.shape
    N = wq.shape[0]
    acc = torch.empty((M, N), dtype=torch.float32, device=xq.device) if acc is None else acc
    need = sq_w8a8_linear_workspace_size(M, N, K)
    if workspace is None:
        workspace = _workspace(need, xq.device, stream)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().sq_w8a8_accumulate_e4m3(_ptr(xq), _ptr(wq), M, N, K, _ptr(acc), acc.stride(0), _ptr(workspace),
                                         wbytes, _stream(stream)), "sq_w8a8_accumulate_e4m3")
    return acc


# Size of the scratch array compiled into libsq.so for the allocation-free
# decode entry point (SQ_DECODE_STATIC_SCRATCH_BYTES in include/sq.h; the
# library reports the value it was built with, sq_decode_static_scratch_bytes).
SQ_DECODE_STATIC_SCRATCH_BYTES = 8 << 20


def sq_decode_static_scratch_bytes() -> int:
    """The scratch size as built into the loaded library."""
    return int(lib().sq_decode_static_scratch_bytes())


def sq_w8a8_linear_decode_noalloc(xq: torch.Tensor, x_scale: torch.Tensor, wq: torch.Tensor,
                                  w_scale: torch.Tensor, out_dtype=torch.bfloat16, y=None,
                                  stream=None) -> torch.Tensor:
    """sq_w8a8_linear for 1 <= M <= 64 without a caller workspace: for callers
    that must not allocate device memory at call time, the library uses a
    scratch array of its own (shared by all calls on a device, so calls must
    not overlap on the GPU).  y may be preallocated to avoid any allocation
    here as well."""
    M, K = xq.shape
    N = wq.shape[0]
    y = torch.empty((M, N), dtype=out_dtype, device=xq.device) if y is None else y
    _rowmajor(y, "y")
    _check(lib().sq_w8a8_linear_decode_noalloc(_ptr(xq), _ptr(x_scale), _ptr(wq), _ptr(w_scale), M, N, K,
                                               _ptr(y), _dtype(y, "y"), y.stride(0), _stream(stream)),
           "sq_w8a8_linear_decode_noalloc")
    return y


def sq_selftest_wait_timeout(limit_ms: int = 100, stream=None) -> int:
    """Runs the bounded-wait self-test kernel (see include/sq.h); returns the
    launch status.  Follow with sq_check_device_error()."""
    return int(lib().sq_selftest_wait_timeout(int(limit_ms), _stream(stream)))


def sq_check_device_error(stream=None) -> int:
    """Synchronises the stream; returns SQ_OK or SQ_ERR_TIMEOUT (and clears it).
    After a timeout the cached workspaces are dropped: a kernel that stopped
    early may have left tile counts in them."""
    status = int(lib().sq_check_device_error(_stream(stream)))
    if status != SQ_OK:
        _WORKSPACES.clear()
    return status

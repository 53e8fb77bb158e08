"""The C ABI without a GPU: the library loads, exports every function the
header declares, and rejects invalid arguments on the host before touching
CUDA (each call below returns before its first CUDA call)."""
import ctypes

import pytest

import w8a8_post_quantization_channel_b200 as sq

INV = sq.SQ_ERR_INVALID_ARG
A16 = 1 << 20          # a fake, 16-byte aligned address (never dereferenced)
MIS = (1 << 20) + 4    # misaligned


def test_library_exports_every_header_function():
    names = sq.header_functions()
    assert {"sq_calib_absmax", "sq_smooth_quant_weight", "sq_quant_act", "sq_w8a8_linear",
            "sq_w8a8_linear_workspace_size", "sq_w8a8_accumulate", "sq_check_device_error",
            "sq_status_string"} <= set(names)
    L = sq.lib()
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    for code in range(5):
        s = sq.sq_status_string(code)
        assert s.startswith("SQ_")
    assert "unknown" in sq.sq_status_string(99)


def test_calib_argument_checks():
    L = sq.lib()
    f = L.sq_calib_absmax
    assert f(A16, sq.SQ_BF16, 0, 256, 256, A16, None) == sq.SQ_OK        # empty stream: no-op
    assert f(None, sq.SQ_BF16, 0, 256, 256, A16, None) == sq.SQ_OK       # x unused when T == 0
    assert f(None, sq.SQ_BF16, 4, 256, 256, A16, None) == INV             # null x
    assert f(A16, sq.SQ_BF16, 4, 256, 256, None, None) == INV             # null amax
    assert f(A16, sq.SQ_BF16, 4, 250, 256, A16, None) == INV              # K % 16
    assert f(A16, sq.SQ_BF16, 4, 256, 255, A16, None) == INV              # ld < K / unaligned rows
    assert f(A16, sq.SQ_BF16, 4, 256, 260, A16, None) == INV              # row stride 520 B not 16-B multiple
    assert f(MIS, sq.SQ_BF16, 4, 256, 256, A16, None) == INV              # misaligned x
    assert f(A16, 7, 4, 256, 256, A16, None) == INV                       # bad dtype
    assert f(A16, sq.SQ_F32, -1, 256, 256, A16, None) == INV              # negative T
    assert f(A16, sq.SQ_F32, 4, 0, 256, A16, None) == INV                 # K == 0


def test_smooth_quant_weight_argument_checks():
    f = sq.lib().sq_smooth_quant_weight
    ok = dict(w=A16, wt=sq.SQ_F16, lay=sq.SQ_W_NK, K=256, N=512, ld=256, amax=A16, alpha=0.5,
              wq=A16, ws=A16, s=A16, inv=A16)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["w"], a["wt"], a["lay"], a["K"], a["N"], a["ld"], a["amax"], ctypes.c_float(a["alpha"]),
                 a["wq"], a["ws"], a["s"], a["inv"], None)

    assert call(alpha=-0.1) == INV
    assert call(alpha=1.5) == INV
    assert call(alpha=float("nan")) == INV
    assert call(lay=3) == INV
    assert call(N=500) == INV
    assert call(K=248) == INV
    assert call(ld=128) == INV                 # NK: ld >= K
    assert call(lay=sq.SQ_W_KN, ld=256) == INV  # KN: ld >= N = 512
    assert call(w=None) == INV
    assert call(wq=None) == INV
    assert call(ws=MIS) == INV
    assert call(s=None) == INV
    assert call(inv=None) == INV
    assert call(amax=None) == INV


def test_quant_act_argument_checks():
    f = sq.lib().sq_quant_act
    assert f(None, sq.SQ_BF16, 0, 256, 256, A16, None, None, None) == sq.SQ_OK
    assert f(A16, sq.SQ_BF16, 8, 256, 256, None, A16, A16, None) == INV
    assert f(A16, sq.SQ_BF16, 8, 256, 256, A16, None, A16, None) == INV
    assert f(A16, sq.SQ_BF16, 8, 256, 256, A16, A16, None, None) == INV
    assert f(A16, sq.SQ_BF16, 8, 24, 24, A16, A16, A16, None) == INV
    assert f(MIS, sq.SQ_F32, 8, 256, 256, A16, A16, A16, None) == INV


def test_scatter_argument_checks_host():
    f = sq.lib().sq_w8a8_linear_scatter
    dsts = (ctypes.c_void_p * 2)(A16, A16 + 4096)
    mis = (ctypes.c_void_p * 2)(A16, MIS)
    assert f(A16, A16, A16, A16, 0, 256, 256, dsts, 2, sq.SQ_BF16, 256, None, 0, None) == sq.SQ_OK  # M == 0
    assert f(A16, A16, A16, A16, 64, 256, 256, None, 2, sq.SQ_BF16, 256, None, 0, None) == INV
    assert f(A16, A16, A16, A16, 64, 256, 256, dsts, 0, sq.SQ_BF16, 256, None, 0, None) == INV
    assert f(A16, A16, A16, A16, 64, 256, 256, dsts, 9, sq.SQ_BF16, 256, None, 0, None) == INV
    assert f(A16, A16, A16, A16, 64, 256, 256, mis, 2, sq.SQ_BF16, 256, None, 0, None) == INV
    assert f(A16, A16, A16, None, 64, 256, 256, dsts, 2, sq.SQ_BF16, 256, None, 0, None) == INV


def test_rotation_argument_checks():
    f = sq.lib().sq_quant_act_rotated
    assert f(None, sq.SQ_BF16, 0, 256, 256, A16, 16, A16, None, None, None) == sq.SQ_OK          # M == 0
    assert f(A16, sq.SQ_BF16, 8, 256, 256, A16, 24, A16, A16, A16, None) == INV                  # n not 2^k
    assert f(A16, sq.SQ_BF16, 8, 256, 256, A16, 1, A16, A16, A16, None) == INV                   # n < 2
    assert f(A16, sq.SQ_BF16, 8, 272, 272, A16, 32, A16, A16, A16, None) == INV                  # K % n
    assert f(A16, sq.SQ_BF16, 8, 16400, 16400, A16, 16, A16, A16, A16, None) == sq.SQ_ERR_UNSUPPORTED   # K
    assert f(A16, sq.SQ_F32, 8, 8208, 8208, A16, 16, A16, A16, A16, None) == sq.SQ_ERR_UNSUPPORTED
    assert f(A16, sq.SQ_BF16, 8, 256, 256, A16, 16, None, A16, A16, None) == INV                 # null table
    g = sq.lib().sq_smooth_quant_weight_rotated
    a = ctypes.c_float(0.5)
    assert g(A16, sq.SQ_BF16, 256, 64, 256, A16, ctypes.c_float(2.0), 16, A16, A16, A16, A16, A16, None) == INV
    assert g(A16, sq.SQ_BF16, 256, 64, 256, A16, a, 12, A16, A16, A16, A16, A16, None) == INV


def test_producer_argument_checks():
    L = sq.lib()
    fold = L.sq_fold_smooth_into_norm
    assert fold(None, A16, 256, A16, None) == INV
    assert fold(A16, None, 256, A16, None) == INV
    assert fold(A16, A16, 256, MIS, None) == INV
    assert fold(A16, A16, 0, A16, None) == INV
    f = L.sq_rmsnorm_quant_act
    eps = ctypes.c_float(1e-5)
    assert f(None, sq.SQ_BF16, 0, 256, 256, A16, eps, None, None, None) == sq.SQ_OK     # M == 0: no-op
    assert f(A16, sq.SQ_BF16, 8, 256, 256, None, eps, A16, A16, None) == INV            # null gs
    assert f(A16, sq.SQ_BF16, 8, 256, 256, A16, ctypes.c_float(-1.0), A16, A16, None) == INV
    assert f(A16, sq.SQ_BF16, 8, 256, 256, A16, ctypes.c_float(float("nan")), A16, A16, None) == INV
    assert f(A16, sq.SQ_BF16, 8, 256, 256, A16, ctypes.c_float(float("inf")), A16, A16, None) == INV
    assert f(A16, sq.SQ_BF16, 8, 24, 24, A16, eps, A16, A16, None) == INV               # K % 16
    assert f(A16, sq.SQ_BF16, 8, 16400, 16400, A16, eps, A16, A16, None) == sq.SQ_ERR_UNSUPPORTED
    assert f(A16, sq.SQ_F32, 8, 8208, 8208, A16, eps, A16, A16, None) == sq.SQ_ERR_UNSUPPORTED
    ln = L.sq_layernorm_quant_act
    assert ln(None, sq.SQ_BF16, 0, 256, 256, A16, None, eps, None, None, None) == sq.SQ_OK   # M == 0: no-op
    assert ln(A16, sq.SQ_BF16, 8, 256, 256, None, A16, eps, A16, A16, None) == INV          # null gs
    assert ln(A16, sq.SQ_BF16, 8, 256, 256, A16, MIS, eps, A16, A16, None) == INV           # misaligned bs
    assert ln(A16, sq.SQ_BF16, 8, 256, 256, A16, A16, ctypes.c_float(0.0), A16, A16, None) == INV  # eps = 0
    assert ln(A16, sq.SQ_BF16, 8, 256, 256, A16, A16, ctypes.c_float(float("nan")), A16, A16, None) == INV
    assert ln(A16, sq.SQ_BF16, 8, 24, 24, A16, A16, eps, A16, A16, None) == INV             # K % 16
    assert ln(A16, sq.SQ_BF16, 8, 256, 200, A16, A16, eps, A16, A16, None) == INV           # ldx < K
    assert ln(A16, sq.SQ_BF16, 8, 16400, 16400, A16, None, eps, A16, A16, None) == sq.SQ_ERR_UNSUPPORTED
    assert ln(A16, sq.SQ_F32, 8, 8208, 8208, A16, None, eps, A16, A16, None) == sq.SQ_ERR_UNSUPPORTED
    st = L.sq_static_act_scale
    assert st(A16, A16, 256, MIS + 1, None) == INV                                       # delta not 4-B aligned
    assert st(None, A16, 256, A16, None) == INV
    qs = L.sq_quant_act_static
    assert qs(None, sq.SQ_F16, 0, 256, 256, A16, A16, None, None, None) == sq.SQ_OK
    assert qs(A16, sq.SQ_F16, 8, 256, 256, A16, None, A16, A16, None) == INV             # null delta
    assert qs(A16, sq.SQ_F16, 8, 256, 256, None, A16, A16, A16, None) == INV             # null inv_s


def test_linear_argument_checks():
    f = sq.lib().sq_w8a8_linear
    base = [A16, A16, A16, A16, 64, 256, 256, A16, sq.SQ_BF16, 256, None, 0, None]

    def call(i, v):
        a = list(base)
        a[i] = v
        return f(*a)

    assert call(4, 0) == sq.SQ_OK          # M == 0: no-op
    assert call(5, 40) == INV              # N % 16
    assert call(6, 40) == INV              # K % 16
    assert call(9, 128) == INV             # ldy < N
    assert call(8, 9) == INV               # bad output dtype
    assert call(0, None) == INV
    assert call(2, None) == INV
    assert call(3, None) == INV
    assert call(7, MIS) == INV
    acc = sq.lib().sq_w8a8_accumulate
    assert acc(A16, A16, 0, 256, 256, A16, 256, None, 0, None) == sq.SQ_OK
    assert acc(A16, A16, 4, 256, 256, None, 256, None, 0, None) == INV
    assert acc(A16, A16, 4, 256, 256, A16, 100, None, 0, None) == INV


def test_fp8_argument_checks():
    L = sq.lib()
    qa = L.sq_quant_act_e4m3
    assert qa(None, sq.SQ_BF16, 0, 256, 256, A16, None, None, None) == sq.SQ_OK     # M == 0: no-op
    assert qa(A16, sq.SQ_BF16, 8, 256, 256, None, A16, A16, None) == INV            # null inv_s
    assert qa(A16, sq.SQ_BF16, 8, 24, 24, A16, A16, A16, None) == INV               # K % 16
    w = L.sq_smooth_quant_weight_e4m3
    assert w(A16, sq.SQ_F16, sq.SQ_W_NK, 256, 512, 256, A16, ctypes.c_float(2.0), A16, A16, A16, A16, None) == INV
    assert w(A16, sq.SQ_F16, sq.SQ_W_NK, 256, 512, 256, None, ctypes.c_float(0.5), A16, A16, A16, A16, None) == INV
    lin = L.sq_w8a8_linear_e4m3
    assert lin(A16, A16, A16, A16, 0, 256, 256, A16, sq.SQ_BF16, 256, None, 0, None) == sq.SQ_OK
    assert lin(A16, A16, A16, A16, 64, 40, 256, A16, sq.SQ_BF16, 256, None, 0, None) == INV   # N % 16
    assert lin(None, A16, A16, A16, 64, 256, 256, A16, sq.SQ_BF16, 256, None, 0, None) == INV
    acc = L.sq_w8a8_accumulate_e4m3
    assert acc(A16, A16, 4, 256, 256, A16, 100, None, 0, None) == INV                  # ldacc < N


def test_decode_noalloc_and_selftest_argument_checks():
    L = sq.lib()
    f = L.sq_w8a8_linear_decode_noalloc
    assert f(A16, A16, A16, A16, 0, 256, 256, A16, sq.SQ_BF16, 256, None) == sq.SQ_OK   # M == 0: no-op
    assert f(A16, A16, A16, A16, 65, 256, 256, A16, sq.SQ_BF16, 256, None) == sq.SQ_ERR_UNSUPPORTED
    assert f(A16, A16, A16, A16, 8, 256, 256, A16, 9, 256, None) == INV                 # output dtype
    assert f(A16, A16, A16, A16, 8, 256, 256, A16, sq.SQ_BF16, 128, None) == INV        # ldy < N
    assert f(A16, A16, None, A16, 8, 256, 256, A16, sq.SQ_BF16, 256, None) == INV       # null wq
    assert f(A16, A16, A16, A16, 8, 256, 256, MIS, sq.SQ_BF16, 256, None) == INV        # misaligned y
    t = L.sq_selftest_wait_timeout
    assert t(0, None) == INV
    assert t(6000, None) == INV


def test_decode_scratch_size_agrees_everywhere():
    # the header's macro, the value built into the library and the binding's
    # constant must be one number
    import os
    import re
    hdr = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "sq.h")
    with open(hdr) as f:
        m = re.search(r"#define SQ_DECODE_STATIC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", f.read())
    assert m is not None
    macro = int(m.group(1)) << int(m.group(2))
    assert sq.sq_decode_static_scratch_bytes() == macro == sq.SQ_DECODE_STATIC_SCRATCH_BYTES


def test_workspace_size_is_defined_for_all_shapes():
    for M in (0, 1, 8, 64, 128, 2048):
        for N, K in ((256, 256), (4096, 4096), (28672, 8192)):
            need = sq.sq_w8a8_linear_workspace_size(M, N, K)
            if 1 <= M <= 64:   # decode-shaped: int32 partial sums + tile counters
                assert need >= M * N * 4 + 4 * ((N + 127) // 128)
                assert need % 256 == 0
            else:
                assert need == 0


def test_linear_requires_workspace_when_needed():
    f = sq.lib().sq_w8a8_linear
    need = sq.sq_w8a8_linear_workspace_size(8, 256, 256)
    assert f(A16, A16, A16, A16, 8, 256, 256, A16, sq.SQ_BF16, 256, None, 0, None) == INV
    assert f(A16, A16, A16, A16, 8, 256, 256, A16, sq.SQ_BF16, 256, A16, need - 1, None) == INV
    assert f(A16, A16, A16, A16, 8, 256, 256, A16, sq.SQ_BF16, 256, MIS, need, None) == INV


def test_binding_rejects_host_tensors():
    import torch
    with pytest.raises(ValueError):
        sq.sq_calib_absmax(torch.zeros(4, 16), torch.zeros(16))

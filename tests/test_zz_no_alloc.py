"""The allocation-free decode entry point, called through the C ABI.

Some callers cannot allocate device memory when they call the linear layer:
a host framework that owns every byte through its own pool, a loop that
cannot afford cudaMalloc's device-wide synchronisation, code running inside
an allocator callback.  For them, sq_w8a8_linear_decode_noalloc uses a
scratch array built into libsq.so where sq_w8a8_linear would need a caller
workspace (the stream-K decode kernel: at most 32 tokens and more 128-row
tiles of Wq than SMs), and no memory at all for the other decode shapes.

These tests check, on two calls in a row that share the scratch, that it
returns bit for bit what the CPU oracle computes (exact int32 product,
dequant, rounding) and what sq_w8a8_linear returns with a workspace; that
the shapes chosen really use the scratch (the size query is positive), one
of them just under the scratch's size; and that it refuses shapes whose need
exceeds that size.  This file is collected last on purpose: it must pass
alone in a fresh process and after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import w8a8_post_quantization_channel_b200 as sq
from w8a8_post_quantization_channel_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
SQ_DT = {torch.float32: sq.SQ_F32, torch.float16: sq.SQ_F16, torch.bfloat16: sq.SQ_BF16}
ORACLE_DT = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}


def _noalloc_c(xq, xs, wq, ws, y):
    """Direct C-ABI call (no Python-side allocation, no workspace)."""
    fn = sq.lib().sq_w8a8_linear_decode_noalloc
    M, K = xq.shape
    N = wq.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(ctypes.c_void_p(xq.data_ptr()), ctypes.c_void_p(xs.data_ptr()), ctypes.c_void_p(wq.data_ptr()),
              ctypes.c_void_p(ws.data_ptr()), M, N, K, ctypes.c_void_p(y.data_ptr()), SQ_DT[y.dtype],
              y.stride(0), stream)


def _bits(y: torch.Tensor) -> np.ndarray:
    y = y.cpu()
    return y.numpy() if y.dtype == torch.float32 else y.view(torch.int16).numpy().view(np.uint16)


def _case(M, N, K, seed):
    g = synth.gen(seed)
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    wq = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    xs = torch.rand(M, generator=g) * 1e-2
    ws = torch.rand(N, generator=g) * 1e-2
    return xq, wq, xs, ws


# Shapes on the scratch (stream-K: M <= 32, N / 128 > the SM count), one
# whose need lies just under the scratch size, and two that need none.
SCRATCH_SHAPES = [(1, 32768, 4096, torch.bfloat16), (16, 20480, 2048, torch.float16),
                  (31, 65024, 256, torch.float32)]
FREE_SHAPES = [(1, 4096, 4096, torch.bfloat16), (37, 11008, 1024, torch.float16)]


@pytest.mark.parametrize("M,N,K,dt", SCRATCH_SHAPES + FREE_SHAPES)
def test_noalloc_matches_the_oracle_on_two_calls(M, N, K, dt):
    need = sq.sq_w8a8_linear_workspace_size(M, N, K)
    assert need <= sq.sq_decode_static_scratch_bytes()
    if (M, N, K, dt) in SCRATCH_SHAPES:
        assert N // 128 > torch.cuda.get_device_properties(0).multi_processor_count
        assert need > 0, "this shape must exercise the shared scratch"
    else:
        assert need == 0
    for call in range(2):  # two calls in a row on the shared scratch, different inputs
        xq, wq, xs, ws = _case(M, N, K, seed=100 * call + M + N)
        y_ref = oracle.round_to(oracle.dequant(oracle.gemm_i8(xq.numpy(), wq.numpy()), xs.numpy(), ws.numpy()),
                                ORACLE_DT[dt])
        xq_d, wq_d, xs_d, ws_d = xq.to(DEV), wq.to(DEV), xs.to(DEV), ws.to(DEV)
        y = torch.full((M, N), float("nan"), dtype=dt, device=DEV)
        assert _noalloc_c(xq_d, xs_d, wq_d, ws_d, y) == sq.SQ_OK
        torch.cuda.synchronize()
        np.testing.assert_array_equal(_bits(y), y_ref)
        # and what the workspace entry point returns
        ref = sq.sq_w8a8_linear(xq_d, xs_d, wq_d, ws_d, dt)
        assert torch.equal(y, ref)
    assert sq.sq_check_device_error() == sq.SQ_OK


def test_noalloc_python_wrapper():
    M, N, K = 8, 32768, 1024
    assert sq.sq_w8a8_linear_workspace_size(M, N, K) > 0
    xq, wq, xs, ws = _case(M, N, K, seed=7)
    y = sq.sq_w8a8_linear_decode_noalloc(xq.to(DEV), xs.to(DEV), wq.to(DEV), ws.to(DEV), torch.bfloat16)
    y_ref = oracle.round_to(oracle.dequant(oracle.gemm_i8(xq.numpy(), wq.numpy()), xs.numpy(), ws.numpy()), "bf16")
    np.testing.assert_array_equal(_bits(y), y_ref)
    assert sq.sq_check_device_error() == sq.SQ_OK


def test_noalloc_rejects_shapes_beyond_its_scratch():
    fn = sq.lib().sq_w8a8_linear_decode_noalloc
    a = ctypes.c_void_p(1 << 20)  # aligned placeholder, never dereferenced on these paths
    # M above the decode range, and a scratch need above the built-in size
    assert fn(a, a, a, a, 65, 4096, 4096, a, sq.SQ_BF16, 4096, None) == sq.SQ_ERR_UNSUPPORTED
    big_n = 65536  # 32 x 65536 x 4 bytes of partial sums, plus tile counters, > 8 MiB
    assert sq.sq_w8a8_linear_workspace_size(32, big_n, 4096) > sq.sq_decode_static_scratch_bytes()
    assert fn(a, a, a, a, 32, big_n, 4096, a, sq.SQ_BF16, big_n, None) == sq.SQ_ERR_UNSUPPORTED
    assert fn(a, a, a, a, 0, 4096, 4096, a, sq.SQ_BF16, 4096, None) == sq.SQ_OK

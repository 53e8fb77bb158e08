"""The allocation-free decode entry point, called through the C ABI.

Some callers cannot allocate device memory when they call the linear layer
(a host framework that owns every byte through its own pool, a loop that
cannot afford cudaMalloc's device-wide synchronisation, code running inside
an allocator callback).  For them, sq_w8a8_linear_decode_noalloc uses a
scratch array built into libsq.so instead of a caller workspace.  These
tests check that it returns what sq_w8a8_linear (with a workspace) returns,
on two calls in a row that share that scratch, and that it refuses shapes
whose scratch need exceeds the built-in size.  This file is collected last
on purpose: it must pass alone in a fresh process and after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import w8a8_post_quantization_channel_b200 as sq
from w8a8_post_quantization_channel_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
SQ_DT = {torch.float32: sq.SQ_F32, torch.float16: sq.SQ_F16, torch.bfloat16: sq.SQ_BF16}


def _codes(shape, seed):
    return torch.randint(-127, 128, shape, generator=synth.gen(seed), dtype=torch.int8).to(DEV)


def _noalloc_c(xq, xs, wq, ws, y):
    """Direct C-ABI call (no Python-side allocation, no workspace)."""
    fn = sq.lib().sq_w8a8_linear_decode_noalloc
    M, K = xq.shape
    N = wq.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(ctypes.c_void_p(xq.data_ptr()), ctypes.c_void_p(xs.data_ptr()), ctypes.c_void_p(wq.data_ptr()),
              ctypes.c_void_p(ws.data_ptr()), M, N, K, ctypes.c_void_p(y.data_ptr()), SQ_DT[y.dtype],
              y.stride(0), stream)


def _assert_close(got: torch.Tensor, ref: torch.Tensor):
    g = got.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    floor = 1e-6 * max(np.abs(r).max(), 1e-30)
    rel = np.abs(g - r) / np.maximum(np.abs(r), floor)
    assert rel.max() <= 1e-2, f"max rel err {rel.max()}"


@pytest.mark.parametrize("M,N,K,dt", [(1, 4096, 4096, torch.bfloat16), (37, 11008, 4096, torch.float16),
                                      (64, 28672, 1024, torch.float32)])
def test_noalloc_matches_workspace_entry_point_on_two_calls(M, N, K, dt):
    for call in range(2):  # two calls in a row on the shared scratch, different inputs
        seed = 100 * call + M
        xq, wq = _codes((M, K), seed), _codes((N, K), seed + 1)
        xs = torch.rand(M, generator=synth.gen(seed + 2)).to(DEV) * 1e-2
        ws = torch.rand(N, generator=synth.gen(seed + 3)).to(DEV) * 1e-2
        ref = sq.sq_w8a8_linear(xq, xs, wq, ws, dt)
        y = torch.full((M, N), float("nan"), dtype=dt, device=DEV)
        assert _noalloc_c(xq, xs, wq, ws, y) == sq.SQ_OK
        torch.cuda.synchronize()
        _assert_close(y, ref)
        assert torch.equal(y, ref)  # same kernel, same inputs: identical bits
    assert sq.sq_check_device_error() == sq.SQ_OK


def test_noalloc_rejects_shapes_beyond_its_scratch():
    fn = sq.lib().sq_w8a8_linear_decode_noalloc
    a = ctypes.c_void_p(1 << 20)  # aligned placeholder, never dereferenced on these paths
    # M above the decode range, and a scratch need above the built-in size
    assert fn(a, a, a, a, 65, 4096, 4096, a, sq.SQ_BF16, 4096, None) == sq.SQ_ERR_UNSUPPORTED
    big_n = 65536  # 64 x 65536 x 4 bytes of partial sums > 8 MiB
    assert sq.sq_w8a8_linear_workspace_size(64, big_n, 4096) > sq.SQ_DECODE_STATIC_SCRATCH_BYTES
    assert fn(a, a, a, a, 64, big_n, 4096, a, sq.SQ_BF16, big_n, None) == sq.SQ_ERR_UNSUPPORTED
    assert fn(a, a, a, a, 0, 4096, 4096, a, sq.SQ_BF16, 4096, None) == sq.SQ_OK

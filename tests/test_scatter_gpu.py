"""The column-parallel linear's multi-destination epilogue, with G ranks
emulated on one GPU: each "rank" computes its column shard of Y and stores
every tile into all G destination tensors (standing in for the peers' Y
buffers, which on several GPUs are peer-mapped pointers).  After all shards,
every destination must equal the CPU oracle's Y (exact int32 product, the
dequant epilogue, rounding to the output type) bit for bit."""
import functools

import numpy as np
import pytest
import torch

import oracle
import w8a8_post_quantization_channel_b200 as sq
from w8a8_post_quantization_channel_b200 import synth
from w8a8_post_quantization_channel_b200.dist import column_shard

pytestmark = pytest.mark.gpu
DEV = "cuda"


# prefill (CTA-pair and single-CTA kernels), decode with the cluster split
# and (shards of 20480 columns: 160 Wq tiles) with the stream-K kernel
SHAPES = [(2048, 4096, 1024), (300, 1024, 272), (16, 4096, 1024), (8, 40960, 256)]


@functools.lru_cache(maxsize=None)
def _case(M, N, K):
    """Seeded codes and scales of one shape, and the oracle's int32 product."""
    g = synth.gen(M + N + K)
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    wq = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    xs = torch.rand(M, generator=g) * 1e-2
    ws = torch.rand(N, generator=g) * 1e-2
    return xq, wq, xs, ws, oracle.gemm_i8(xq.numpy(), wq.numpy())


def _bits(y: torch.Tensor) -> np.ndarray:
    y = y.cpu()
    return y.numpy() if y.dtype == torch.float32 else y.view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_scatter_to_every_rank_equals_the_oracle(M, N, K, G, out):
    xq, wq, xs, ws, acc = _case(M, N, K)
    y_ref = oracle.round_to(oracle.dequant(acc, xs.numpy(), ws.numpy()), "bf16" if out == torch.bfloat16 else "f32")
    xq_d, wq_d, xs_d, ws_d = xq.to(DEV), wq.to(DEV), xs.to(DEV), ws.to(DEV)
    ys = [torch.full((M, N), -7.0, dtype=out, device=DEV) for _ in range(G)]
    for r in range(G):
        n0, n1 = column_shard(N, G, r)
        if n1 > n0:
            sq.sq_w8a8_linear_scatter(xq_d, xs_d, wq_d[n0:n1].contiguous(), ws_d[n0:n1].contiguous(), ys, n0)
    for y in ys:
        np.testing.assert_array_equal(_bits(y), y_ref)
    assert sq.sq_check_device_error() == sq.SQ_OK


def test_scatter_argument_checks():
    xq = torch.zeros(4, 32, dtype=torch.int8, device=DEV)
    wq = torch.zeros(16, 32, dtype=torch.int8, device=DEV)
    xs = torch.ones(4, device=DEV)
    ws = torch.ones(16, device=DEV)
    ys = [torch.zeros(4, 64, dtype=torch.bfloat16, device=DEV) for _ in range(9)]
    with pytest.raises(ValueError):
        sq.sq_w8a8_linear_scatter(xq, xs, wq, ws, ys, 0)          # more than 8 destinations
    with pytest.raises(ValueError):
        sq.sq_w8a8_linear_scatter(xq, xs, wq, ws, ys[:2], 56)     # shard past the last column
    with pytest.raises(sq.SqError):
        sq.sq_w8a8_linear_scatter(xq, xs, wq, ws, ys[:2], 4)      # column 4 of bf16: not 16-byte aligned

"""The column-parallel linear's multi-destination epilogue, with G ranks
emulated on one GPU: each "rank" computes its column shard of Y and stores
every tile into all G destination tensors (standing in for the peers' Y
buffers, which on several GPUs are peer-mapped pointers).  After all shards,
every destination must equal the single-GPU linear bit for bit."""
import pytest
import torch

import w8a8_post_quantization_channel_b200 as sq
from w8a8_post_quantization_channel_b200.dist import column_shard

pytestmark = pytest.mark.gpu
DEV = "cuda"


# prefill (CTA-pair and single-CTA kernels), decode with the cluster split
# and (shards of 20480 columns: 160 Wq tiles) with the stream-K kernel
SHAPES = [(2048, 4096, 1024), (300, 1024, 272), (16, 4096, 1024), (8, 40960, 256)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_scatter_to_every_rank_equals_the_linear(M, N, K, G, out):
    g = torch.Generator(device=DEV).manual_seed(M + N + K + G)
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8, device=DEV)
    wq = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8, device=DEV)
    xs = torch.rand(M, generator=g, device=DEV) * 1e-2
    ws = torch.rand(N, generator=g, device=DEV) * 1e-2
    y_full = sq.sq_w8a8_linear(xq, xs, wq, ws, out)
    ys = [torch.full((M, N), -7.0, dtype=out, device=DEV) for _ in range(G)]
    for r in range(G):
        n0, n1 = column_shard(N, G, r)
        if n1 > n0:
            sq.sq_w8a8_linear_scatter(xq, xs, wq[n0:n1].contiguous(), ws[n0:n1].contiguous(), ys, n0)
    for y in ys:
        assert torch.equal(y, y_full)
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

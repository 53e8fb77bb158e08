"""Data-parallel calibration across ranks, on CPU with gloo (world size 2).

Calibration is a per-channel maximum over tokens, so ranks that calibrate on
disjoint shards and merge with an element-wise MAX all-reduce must reproduce
the single-process maxima bit for bit; the smoothing factors and INT8
weights that follow are then identical on every rank.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from w8a8_post_quantization_channel_b200.dist import allreduce_amax, column_parallel_linear, column_shard, shard_range


def test_shard_range_partitions():
    for total in (0, 1, 7, 64, 65536, 65537):
        for world in (1, 2, 3, 8):
            spans = [shard_range(total, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(10, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        import oracle
        from w8a8_post_quantization_channel_b200 import synth
        T, K, N = 1000, 272, 64
        o = synth.outliers(K, frac=0.02, mult=100.0, seed=5)
        stream = synth.activations(T, K, o, seed=6, dtype=torch.bfloat16).float().numpy()
        a, b = shard_range(T, world, rank)
        local = torch.from_numpy(oracle.calib_absmax(stream[a:b]))
        merged = allreduce_amax(local.clone())
        full = oracle.calib_absmax(stream)
        ok_amax = np.array_equal(merged.numpy(), full)
        # the weights every rank derives from the merged maxima are identical
        w = synth.weights(K, N, 7, torch.float32, "nk").numpy()
        s, _ = oracle.smooth_factor(merged.numpy(), oracle.weight_absmax(w, oracle.LAYOUT_NK), 0.5)
        wq, _ = oracle.smooth_quant_weight(w, oracle.LAYOUT_NK, s)
        digest = torch.tensor([int(wq.astype(np.int64).sum()), int((wq.astype(np.int64) ** 2).sum())])
        gathered = [torch.zeros_like(digest) for _ in range(world)]
        dist.all_gather(gathered, digest)
        ok_w = all(torch.equal(g, gathered[0]) for g in gathered)
        # a rank's own shard alone is (generally) not enough
        partial_differs = not np.array_equal(local.numpy(), full)
        q.put((rank, ok_amax, ok_w, partial_differs))
        dist.destroy_process_group()
    except Exception as e:  # pragma: no cover
        q.put((rank, repr(e), False, False))


def test_two_rank_calibration_merge_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    for rank, ok_amax, ok_w, partial_differs in results:
        assert ok_amax is True, f"rank {rank}: {ok_amax}"
        assert ok_w
    assert any(r[3] for r in results)


def test_column_shard_partitions():
    for n in (16, 48, 4096, 12288, 28672):
        for world in (1, 2, 3, 4, 8):
            spans = [column_shard(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c
            assert all(a % 16 == 0 and b % 16 == 0 for a, b in spans)
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 16
    with pytest.raises(ValueError):
        column_shard(100, 2, 0)


def _oracle_linear(xq, x_scale, wq, w_scale, out_dtype):
    import oracle
    acc = oracle.gemm_i8(xq.numpy(), wq.numpy())
    return torch.from_numpy(oracle.dequant(acc, x_scale.numpy(), w_scale.numpy()))


def _column_worker(rank, world, port, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        import oracle
        M, K, N = 24, 64, 48
        g = torch.Generator().manual_seed(11)
        xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
        wq = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
        xs = torch.rand(M, generator=g) * 1e-2
        ws = torch.rand(N, generator=g) * 1e-2
        n0, n1 = column_shard(N, world, rank)
        y = column_parallel_linear(xq, xs, wq[n0:n1].contiguous(), ws[n0:n1].contiguous(), N,
                                   out_dtype=torch.float32, linear=_oracle_linear)
        full = oracle.dequant(oracle.gemm_i8(xq.numpy(), wq.numpy()), xs.numpy(), ws.numpy())
        q.put((rank, bool(np.array_equal(y.numpy(), full)), n1 - n0))
        dist.destroy_process_group()
    except Exception as e:  # pragma: no cover
        q.put((rank, repr(e), -1))


@pytest.mark.parametrize("world", [2, 4])
def test_column_parallel_linear_gathers_every_shard_gloo(world):
    # N = 48 over 4 ranks leaves the last rank without columns
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_column_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert all(ok is True for _, ok, _ in results), results
    assert sum(w for _, _, w in results) == 48


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

from w8a8_post_quantization_channel_b200.dist import allreduce_amax, shard_range


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

"""The data-parallel host path on CPU: two gloo ranks, no GPU.

Each rank takes its share of a token batch, computes the float64 oracle
gradients of its share, and the all-reduce of dA and dB must give the
gradients of the whole batch (both are sums over tokens).  Also checks the
max-over-ranks timing helper and the token split."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_nf4_quantized_07_b200 import dp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from oracle import linear
        g = np.random.Generator(np.random.PCG64(5))
        n, din, dout, r, s = 37, 48, 40, 4, 1.5
        Wp = g.standard_normal((dout, din)) * 0.1
        X = g.standard_normal((n, din))
        A = g.standard_normal((r, din)) * 0.3
        B = g.standard_normal((dout, r)) * 0.3
        dY = g.standard_normal((n, dout))
        t0, t1 = dp.token_range(n, world, rank)
        _, dA, dB = linear.backward(Wp, X[t0:t1], A, B, s, dY[t0:t1])
        tA, tB = torch.from_numpy(dA.copy()), torch.from_numpy(dB.copy())
        dp.allreduce_adapter_grads(tA, tB)
        _, dA_full, dB_full = linear.backward(Wp, X, A, B, s, dY)
        ok = np.allclose(tA.numpy(), dA_full, rtol=1e-12, atol=1e-12) and \
            np.allclose(tB.numpy(), dB_full, rtol=1e-12, atol=1e-12)
        mx = dp.max_over_ranks(10.0 + rank)
        q.put((rank, ok, mx, (t0, t1)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_token_range_partitions_the_batch():
    for n in (1, 7, 64, 2049):
        for world in (1, 2, 3, 8):
            ranges = [dp.token_range(n, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1


def test_two_rank_gloo_allreduce_equals_full_batch_gradients():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    assert [r[1] for r in results] == [True, True]
    assert [r[2] for r in results] == [11.0, 11.0]
    assert results[0][3] == (0, 19) and results[1][3] == (19, 37)

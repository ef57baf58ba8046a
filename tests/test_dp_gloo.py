"""The data-parallel host path on CPU: two gloo ranks, no GPU.

Each rank takes its share of a token batch, computes the float64 oracle
gradients of its share, and the all-reduce of dA and dB must give the
gradients of the whole batch (both are sums over tokens).  Also checks the
max-over-ranks timing helper, the token split, and the rank wiring that
bench.py's training step uses (dp.init_from_env, dp.train_step, dp.barrier,
dp.finish): a few training steps on two ranks leave both replicas of A and B
identical and equal to full-batch training on one process."""
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


STEPS, LR = 3, 1e-2


def _problem():
    g = np.random.Generator(np.random.PCG64(6))
    n, din, dout, r, s = 29, 40, 24, 4, 2.0
    return (g.standard_normal((dout, din)) * 0.1, g.standard_normal((n, din)), g.standard_normal((r, din)) * 0.3,
            g.standard_normal((dout, r)) * 0.3, [g.standard_normal((n, dout)) for _ in range(STEPS)], s)


def _train(Wp, X, A, B, dYs, s, t0, t1, world):
    """STEPS AdamW steps of A and B on tokens [t0, t1) through dp.train_step
    (the oracle's backward and AdamW stand in for the kernels)."""
    from oracle import adamw, linear
    A, B = A.copy(), B.copy()
    dA, dB = torch.zeros(A.shape, dtype=torch.float64), torch.zeros(B.shape, dtype=torch.float64)
    mA, vA, mB, vB = (np.zeros_like(A), np.zeros_like(A), np.zeros_like(B), np.zeros_like(B))
    for k in range(STEPS):
        def backward():
            _, gA, gB = linear.backward(Wp, X[t0:t1], A, B, s, dYs[k][t0:t1])
            dA.copy_(torch.from_numpy(gA))
            dB.copy_(torch.from_numpy(gB))

        def update():
            nonlocal A, B, mA, vA, mB, vB
            A, mA, vA = adamw.adamw_step(A, dA.numpy(), mA, vA, k + 1, LR)
            B, mB, vB = adamw.adamw_step(B, dB.numpy(), mB, vB, k + 1, LR)
        dp.train_step(backward, update, dA, dB, world)
    return A, B


def _train_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    rk, wd, local = dp.init_from_env("cpu", timeout_s=60.0)
    try:
        Wp, X, A, B, dYs, s = _problem()
        t0, t1 = dp.token_range(X.shape[0], wd, rk)
        A1, B1 = _train(Wp, X, A, B, dYs, s, t0, t1, wd)
        dp.barrier(wd)
        q.put((rk, wd, local, A1, B1))
    finally:
        dp.finish(wd)


def test_two_rank_training_steps_keep_replicas_equal_to_full_batch_training():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_train_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted([q.get(timeout=120) for _ in range(world)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [(r[0], r[1], r[2]) for r in results] == [(0, 2, 0), (1, 2, 1)]
    (_, _, _, A0, B0), (_, _, _, A1, B1) = results
    assert np.array_equal(A0, A1) and np.array_equal(B0, B1), "the replicas diverged"
    Wp, X, A, B, dYs, s = _problem()
    Af, Bf = _train(Wp, X, A, B, dYs, s, 0, X.shape[0], 1)  # one process, the whole batch
    assert not np.allclose(Af, A) and not np.allclose(Bf, B)  # the steps moved the factors
    np.testing.assert_allclose(A0, Af, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(B0, Bf, rtol=1e-10, atol=1e-12)


def test_single_rank_wiring_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert dp.init_from_env("cpu") == (0, 1, 0)
    assert not dist.is_initialized()
    Wp, X, A, B, dYs, s = _problem()
    A1, B1 = _train(Wp, X, A, B, dYs, s, 0, X.shape[0], 1)
    dp.barrier(1)
    dp.finish(1)
    assert A1.shape == A.shape and B1.shape == B.shape

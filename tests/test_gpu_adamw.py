"""GPU parity of the paged AdamW step (qln_adamw_step) against the float64
oracle, with the states in device memory, in managed (unified) memory paged
in and out, and replayed from a CUDA graph with a device-side step counter.

Tolerance (derived from fp32 evaluation, ~6 rounded operations per element,
compounded over the steps of a test).  m = b1 m + (1 - b1) g can cancel, so
its rounding error is relative to the magnitudes that enter it: with the
envelope mabs = b1 mabs + (1 - b1) |g| (float64, from zero),
  |m - m*| <= 4e-6 mabs,  |v - v*| <= 4e-6 v*  (v never cancels),
  |p - p*| <= 4e-6 (|p*| + 4 lr)  (the step is at most a few lr),
and the BF16 copy equals RN(the fp32 master) exactly."""
import ctypes

import numpy as np
import pytest
import torch

from bit_nf4_quantized_07_b200 import api
from oracle import adamw

pytestmark = pytest.mark.gpu
HP = dict(lr=2e-3, betas=(0.9, 0.995), eps=1e-8, weight_decay=0.01)


def _data(n, seed):
    g = np.random.Generator(np.random.PCG64(seed))
    p0 = (g.standard_normal(n) * 0.02).astype(np.float32)
    grads = [(g.standard_normal(n) * 10 ** g.uniform(-5, -1)).astype(np.float32) for _ in range(5)]
    return p0, grads


def _check(p, m, v, pr, mr, vr, mabs, lr):
    assert np.all(np.abs(p - pr) <= 4e-6 * (np.abs(pr) + 4 * lr)), np.max(np.abs(p - pr))
    assert np.all(np.abs(m - mr) <= 4e-6 * mabs + 1e-30), np.max(np.abs(m - mr) / (mabs + 1e-30))
    assert np.all(np.abs(v - vr) <= 4e-6 * vr + 1e-30), np.max(np.abs(v - vr) / (vr + 1e-30))


@pytest.mark.parametrize("n", [1, 3, 64, 4096 + 3, 16 * (4096 + 11008)])
def test_adamw_matches_oracle_over_five_steps(n):
    p0, grads = _data(n, 40 + n % 97)
    p = torch.from_numpy(p0.copy()).cuda()
    m = torch.zeros(n, device="cuda")
    v = torch.zeros(n, device="cuda")
    pb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    step = torch.zeros(1, dtype=torch.int64, device="cuda")
    pr, mr, vr, mabs = p0.astype(np.float64), np.zeros(n), np.zeros(n), np.zeros(n)
    for t in range(1, 6):
        step.fill_(t)
        api.adamw_step(p, torch.from_numpy(grads[t - 1]).cuda(), m, v, step, HP["lr"], HP["betas"], HP["eps"],
                       HP["weight_decay"], param_bf16=pb)
        pr, mr, vr = adamw.adamw_step(pr, grads[t - 1], mr, vr, t, HP["lr"], *HP["betas"], HP["eps"],
                                      HP["weight_decay"])
        mabs = HP["betas"][0] * mabs + (1 - HP["betas"][0]) * np.abs(grads[t - 1].astype(np.float64))
        torch.cuda.synchronize()
        _check(p.cpu().numpy(), m.cpu().numpy(), v.cpu().numpy(), pr, mr, vr, mabs, HP["lr"])
        assert torch.equal(pb, p.to(torch.bfloat16))


def _managed(n):
    from cuda.bindings import runtime as cudart
    err, ptr = cudart.cudaMallocManaged(4 * n, cudart.cudaMemAttachGlobal)
    assert err == cudart.cudaError_t.cudaSuccess
    arr = np.ctypeslib.as_array(ctypes.cast(int(ptr), ctypes.POINTER(ctypes.c_float)), shape=(n,))
    arr[:] = 0.0
    return int(ptr), arr


def test_adamw_with_managed_states_paged_in_and_out():
    """m and v in unified memory, prefetched to the GPU for the update and back
    to host RAM after it: the same bits as with device-memory states."""
    from cuda.bindings import runtime as cudart
    n = 16 * (4096 + 11008)
    p0, grads = _data(n, 7)
    mp, marr = _managed(n)
    vp, varr = _managed(n)
    p = torch.from_numpy(p0.copy()).cuda()
    p_ref = torch.from_numpy(p0.copy()).cuda()
    m_ref = torch.zeros(n, device="cuda")
    v_ref = torch.zeros(n, device="cuda")
    step = torch.zeros(1, dtype=torch.int64, device="cuda")
    cfg = api.CAdamWConfig(HP["lr"], HP["betas"][0], HP["betas"][1], HP["eps"], HP["weight_decay"])
    L = api.lib()
    try:
        for t in range(1, 4):
            step.fill_(t)
            g = torch.from_numpy(grads[t - 1]).cuda()
            st = L.qln_adamw_step(ctypes.c_void_p(p.data_ptr()), ctypes.c_void_p(g.data_ptr()), ctypes.c_void_p(mp),
                                  ctypes.c_void_p(vp), None, n, ctypes.byref(cfg), ctypes.c_void_p(step.data_ptr()),
                                  api.ADAMW_PAGE_IN | api.ADAMW_PAGE_OUT, api._stream())
            assert st == 0, api.status_str(st)
            api.adamw_step(p_ref, g, m_ref, v_ref, step, HP["lr"], HP["betas"], HP["eps"], HP["weight_decay"])
            torch.cuda.synchronize()
            assert np.array_equal(marr, m_ref.cpu().numpy()) and np.array_equal(varr, v_ref.cpu().numpy())
            assert torch.equal(p, p_ref)
    finally:
        cudart.cudaFree(mp)
        cudart.cudaFree(vp)


def test_adamw_graph_replay_reads_the_device_step():
    """One captured step, replayed three times while the graph itself
    increments the device step counter, equals three eager steps."""
    n = 4096 + 5
    p0, grads = _data(n, 9)
    g = torch.from_numpy(grads[0]).cuda()
    pa, ma, va = torch.from_numpy(p0.copy()).cuda(), torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    pe, me, ve = pa.clone(), ma.clone(), va.clone()
    step_a = torch.zeros(1, dtype=torch.int64, device="cuda")
    step_e = torch.zeros(1, dtype=torch.int64, device="cuda")

    def body():
        step_a.add_(1)
        api.adamw_step(pa, g, ma, va, step_a, HP["lr"], HP["betas"], HP["eps"], HP["weight_decay"])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        body()
    for _ in range(3):
        graph.replay()
    for t in range(1, 4):
        step_e.fill_(t)
        api.adamw_step(pe, g, me, ve, step_e, HP["lr"], HP["betas"], HP["eps"], HP["weight_decay"])
    torch.cuda.synchronize()
    assert int(step_a.item()) == 3
    assert torch.equal(pa, pe) and torch.equal(ma, me) and torch.equal(va, ve)

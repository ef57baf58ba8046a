"""The algorithmic FLOP and byte counts behind the bench's rates, checked
against brute-force counts on tiny shapes and against the workload figures
they are quoted with (no GPU)."""
import itertools

import numpy as np
import pytest

import bench
from bit_nf4_quantized_07_b200 import synthetic


def _gemm_macs(m, k, n):
    """Multiply-adds of an (m x k) by (k x n) product, counted one by one."""
    return sum(1 for _ in itertools.product(range(m), range(n), range(k)))


@pytest.mark.parametrize("dout,din,n,r", [(4, 5, 3, 2), (6, 2, 1, 3), (3, 7, 4, 1)])
def test_linear_flops_equal_counted_multiply_adds(dout, din, n, r):
    """Forward: Y = X W'^T (n x din x dout), U = X A^T (n x din x r),
    U B^T (n x r x dout).  Backward: dX = dY W' (n x dout x din),
    G = dY B (n x dout x r), dX += G A (n x r x din), dA = G^T X
    (r x n x din), dB = dY^T U (dout x n x r).  Two FLOPs per multiply-add."""
    cfg = synthetic.LinearConfig("tiny", 0, dout, din, n, r, 1.0, 0.02, 0.02)
    fwd = _gemm_macs(n, din, dout) + _gemm_macs(n, din, r) + _gemm_macs(n, r, dout)
    bwd = (_gemm_macs(n, dout, din) + _gemm_macs(n, dout, r) + _gemm_macs(n, r, din) + _gemm_macs(r, n, din)
           + _gemm_macs(dout, n, r))
    assert cfg.fwd_flops() == 2 * fwd
    assert cfg.bwd_flops() == 2 * bwd


def test_workload_flops_match_the_quoted_figures():
    """Prefill 11008 x 4096, n = 2048, r = 16: 185.7 / 186.7 GFLOP;
    Large 28672 x 8192, n = 4096, r = 64: 1.9435 / 1.9628 TFLOP."""
    p, g = synthetic.PREFILL, synthetic.LARGE
    assert (p.dout, p.din, p.n, p.r) == (11008, 4096, 2048, 16)
    assert (g.dout, g.din, g.n, g.r) == (28672, 8192, 4096, 64)
    assert abs(p.fwd_flops() / 1e9 - 185.7) < 0.05
    assert abs(p.bwd_flops() / 1e9 - 186.7) < 0.05
    assert abs(g.fwd_flops() / 1e12 - 1.9435) < 5e-5
    assert abs(g.bwd_flops() / 1e12 - 1.9628) < 5e-5


def test_codec_bytes_per_param_equal_the_arrays_moved():
    """Quantize + DQ reads fp32 W and writes codes, rhat and one fp32 scale per
    group of 256 blocks; dequant reads those three and writes BF16 W'.  The
    per-parameter counts must equal the sizes of those arrays."""
    rows, cols = 256, 1024  # a whole number of DQ groups
    numel = rows * cols
    nb, ng = numel // 64, numel // (64 * 256)
    w = np.zeros(numel, np.float32)
    codes = np.zeros(numel // 2, np.uint8)
    qabs = np.zeros(nb, np.int8)
    scale = np.zeros(ng, np.float32)
    out = np.zeros(numel, np.uint16)
    q, d = bench.codec_bytes_per_param()
    assert q * numel == pytest.approx(w.nbytes + codes.nbytes + qabs.nbytes + scale.nbytes, rel=1e-12)
    assert d * numel == pytest.approx(codes.nbytes + qabs.nbytes + scale.nbytes + out.nbytes, rel=1e-12)


def test_sweep_size_and_bytes():
    """Every linear of a 32-layer d = 4096, ffn = 11008 decoder: 6,476,005,376
    parameters; 29.25 GB for quantize + DQ and 16.29 GB for dequant."""
    params = synthetic.sweep_params()
    assert params == 32 * (4 * 4096 * 4096 + 3 * 4096 * 11008) == 6_476_005_376
    q, d = bench.codec_bytes_per_param()
    assert abs(q * params / 1e9 - 29.25) < 0.01  # 29.2448 GB, quoted to four figures
    assert abs(d * params / 1e9 - 16.29) < 0.01


def test_decode_bytes_per_call():
    """Decode layer 4096 x 4096, r = 16: 8.93 / 8.98 / 9.18 MB per call at
    n = 1 / 4 / 16, of which the weight is 8.65 MB (codes 8.39 MB, rhat
    0.26 MB, scales 4 KB); the parts are the sizes of the arrays read and
    written."""
    rows = cols = 4096
    r = 16
    weight = rows * cols // 2 + rows * cols // 64 + 4 * (rows * cols // (64 * 256)) + 4
    assert abs(weight / 1e6 - 8.65) < 0.005
    for n, mb in ((1, 8.93), (4, 8.98), (16, 9.18)):
        acts = 2 * (n * cols + r * cols + rows * r + n * r + n * rows)
        got = bench.decode_bytes_per_call(rows, cols, n, r)
        assert got == weight + acts
        assert abs(got / 1e6 - mb) < 0.005

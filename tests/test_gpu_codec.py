"""GPU parity of the codec kernels (quantize, double quantization, dequant)
against the CPU oracle: bit-exact codes, constants, mean and BF16 weights."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_07_b200 import api, synthetic
from oracle import codec
from tests.oracle_ref import dev_bf16_bits

pytestmark = pytest.mark.gpu


def _gpu_codec(w: np.ndarray):
    W = torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda()
    rows, cols = w.reshape(-1, 64).shape[0], 64
    codes, absmax = api.nf4_quantize(W)
    qabs, scale, mu = api.nf4_double_quant(absmax)
    wq = api.NF4Weight(codes=codes, rows=rows, cols=cols, absmax=absmax, qabs=qabs, dq_scale=scale, dq_mean=mu)
    deq = api.nf4_dequant(wq)
    wplain = api.NF4Weight(codes=codes, rows=rows, cols=cols, absmax=absmax)
    deq_plain = api.nf4_dequant(wplain)
    torch.cuda.synchronize()
    return (codes.cpu().numpy(), absmax.cpu().numpy(), qabs.cpu().numpy(), scale.cpu().numpy(),
            mu.cpu().numpy()[0], dev_bf16_bits(deq).reshape(-1), dev_bf16_bits(deq_plain).reshape(-1))


def _check_all(w):
    n = w.size
    g = _gpu_codec(w)
    codes, absmax = codec.quantize(w)
    qabs, scale, mu = codec.double_quant(absmax)
    assert np.array_equal(g[1].view(np.uint32), absmax.view(np.uint32)), "absmax"
    assert np.array_equal(g[0], codes), f"codes: {np.sum(g[0] != codes)} bytes differ"
    assert np.float32(g[4]).view(np.uint32) == np.float32(mu).view(np.uint32), (g[4], mu)
    assert np.array_equal(g[3].view(np.uint32), scale.view(np.uint32)), "dq scale"
    assert np.array_equal(g[2], qabs), "dq codes"
    assert np.array_equal(g[5], codec.dequant(codes, n, qabs=qabs, scale=scale, mu=mu)), "dequant (DQ)"
    assert np.array_equal(g[6], codec.dequant(codes, n, absmax=absmax)), "dequant (plain)"


@pytest.mark.parametrize("shape,seed", [((512, 512), 1), ((1, 64), 2), ((3, 320), 3), ((77, 192), 4),
                                        ((1000, 192), 5), ((257, 256), 6), ((4096, 4096), 7)])
def test_codec_bit_exact(shape, seed):
    _check_all(synthetic.normal_f32(shape, 0.02, seed))


def test_codec_crafted_edge_blocks():
    cb = codec.cb32()
    blocks = []
    blocks.append(np.zeros(64, np.float32))                              # all zero
    b = np.zeros(64, np.float32); b[17] = -5.0; blocks.append(b)          # single nonzero
    blocks.append(np.full(64, -0.0, np.float32))                          # negative zeros
    b = np.zeros(64, np.float32); b[0], b[1] = 2.0, -2.0; blocks.append(b)  # +-absmax tie
    blocks.append(np.tile(np.r_[cb, cb[::-1]], 2).astype(np.float32) * np.float32(0.37))  # every code
    for k in range(15):                                                   # near/at every midpoint
        mid = (float(cb[k]) + float(cb[k + 1])) / 2
        m32 = np.float32(mid)
        b = np.full(64, m32, np.float32)
        b[0] = 1.0
        b[1:8] = np.nextafter(m32, np.float32(-2))
        b[8:16] = np.nextafter(m32, np.float32(2))
        b[16:24] = np.nextafter(np.nextafter(m32, np.float32(2)), np.float32(2))
        blocks.append(b)
    blocks.append(np.float32(1e-38) * np.linspace(-1, 1, 64, dtype=np.float32))   # subnormal-range block
    blocks.append(np.float32(3e38) * np.linspace(-1, 1, 64, dtype=np.float32))    # near fp32 max
    w = np.concatenate(blocks)
    _check_all(w)


def test_dq_degenerate_groups():
    w = np.tile(np.r_[np.float32(0.25), np.zeros(63, np.float32)], 600)   # all a_j equal -> b == 0
    _check_all(w)


def test_prefill_size_codec_bit_exact():
    cfg = synthetic.PREFILL
    _check_all(synthetic.weight_f32(cfg))


@pytest.mark.slow
def test_large_size_codec_sampled():
    """Full Large weight (28672 x 8192, 0.1 % x10 outliers) on the GPU; the
    oracle checks 8192 sampled blocks plus the first and last, the full absmax
    (NumPy max) and the full double quantization."""
    cfg = synthetic.LARGE
    w = synthetic.weight_f32(cfg)
    codes_g, absmax_g, qabs_g, scale_g, mu_g, deq_g, _ = _gpu_codec(w)
    wb = w.reshape(-1, 64)
    nb = wb.shape[0]
    assert np.array_equal(absmax_g, np.max(np.abs(wb), axis=1))
    qabs, scale, mu = codec.double_quant(absmax_g)
    assert np.float32(mu_g).view(np.uint32) == np.float32(mu).view(np.uint32)
    assert np.array_equal(qabs_g, qabs) and np.array_equal(scale_g.view(np.uint32), scale.view(np.uint32))
    rng = np.random.Generator(np.random.PCG64(99))
    idx = np.unique(np.r_[0, nb - 1, rng.integers(0, nb, 8192)])
    codes_s, _ = codec.quantize(wb[idx])
    assert np.array_equal(codes_g.reshape(nb, 32)[idx], codes_s.reshape(-1, 32))
    # dequant of the sampled blocks with the full-tensor DQ constants
    deq = deq_g.reshape(nb, 64)[idx]
    for k, j in enumerate(idx[:512]):
        ah = codec.dq_restore(qabs[j:j + 1], scale[j // 256:j // 256 + 1], mu)[0]
        ref = codec.dequant(codes_s.reshape(-1, 32)[k], 64, absmax=np.array([ah], np.float32))
        assert np.array_equal(deq[k], ref)

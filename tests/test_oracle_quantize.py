"""Pins of the oracle's blockwise NF4 quantization.

Sources: jjjymmm.cn 2024/03 QLoRA post, "4-bit NormalFloat(NF4)" (divide by
the block ABSMAX, take the closest quant-book value; dequant = table value);
"LoRA 与 QLoRA", QLoRA section 2 (a_j = max|W_j| over 64-weight blocks).
"""
import numpy as np
import pytest

from bit_nf4_quantized_07_b200 import synthetic
from oracle import codec
from tests.conftest import read_golden_values

PRINTED = np.array([float(v) for v in read_golden_values("nf4_codebook_printed.txt")], np.float64)


def _x_of(w):
    """x = fp32(w / a_j) by NumPy's IEEE binary32 division (independent of the C oracle)."""
    w = w.reshape(-1, 64).astype(np.float32)
    a = np.max(np.abs(w), axis=1, keepdims=True)
    with np.errstate(invalid="ignore", divide="ignore"):
        x = np.where(a > 0, w / a, np.float32(0.0)).astype(np.float32)
    return x, a[:, 0]


def test_nearest_against_printed_table():
    # x values at least 2e-4 away from every printed midpoint: the 4-decimal
    # table decides the nearest entry unambiguously.
    mids = (PRINTED[:-1] + PRINTED[1:]) / 2
    g = np.random.Generator(np.random.PCG64(7))
    xs = g.uniform(-1, 1, 20000).astype(np.float32)
    xs = xs[np.min(np.abs(xs[:, None].astype(np.float64) - mids[None, :]), axis=1) > 2e-4]
    for x in xs[:4000]:
        want = int(np.argmin(np.abs(PRINTED - float(x))))
        assert codec.nearest(float(x)) == want


def test_quantize_is_nearest_code_for_every_element():
    w = synthetic.normal_f32((64, 1024), 0.02, 11)
    codes, absmax = codec.quantize(w)
    q = codec.unpack_codes(codes, w.size).reshape(-1, 64)
    x, a = _x_of(w)
    assert np.array_equal(absmax, a)
    _, cb = codec.codebook()
    d = np.abs(x[..., None].astype(np.float64) - cb.astype(np.float64))  # [blk, 64, 16]
    dq = np.take_along_axis(d, q[..., None].astype(np.int64), axis=-1)[..., 0]
    assert np.all(dq <= d.min(axis=-1)), "chosen code is a nearest entry"
    # ties keep the lower index: the first minimum
    assert np.array_equal(q, np.argmin(d, axis=-1))


def test_absmax_element_gets_an_end_code_and_error_bound():
    w = synthetic.normal_f32((128, 512), 0.02, 12)
    codes, absmax = codec.quantize(w)
    q = codec.unpack_codes(codes, w.size).reshape(-1, 64)
    wb = w.reshape(-1, 64)
    i = np.argmax(np.abs(wb), axis=1)
    qa = q[np.arange(q.shape[0]), i]
    assert np.all((qa == 0) | (qa == 15))
    assert np.all(np.where(wb[np.arange(q.shape[0]), i] < 0, qa == 0, qa == 15))
    _, cb = codec.codebook()
    rec = absmax[:, None].astype(np.float64) * cb[q].astype(np.float64)
    gaps = np.diff(cb.astype(np.float64))
    assert gaps.argmax() == 0                     # widest gap: -1 .. -0.6962
    widest = gaps.max() / 2.0
    assert np.all(np.abs(wb - rec) <= absmax[:, None] * (widest + 1e-6))


def test_every_code_appears_on_gaussian_input():
    w = synthetic.normal_f32((256, 1024), 0.02, 13)
    codes, _ = codec.quantize(w)
    assert set(np.unique(codec.unpack_codes(codes, w.size)).tolist()) == set(range(16))


def test_edge_blocks():
    w = np.zeros((4, 64), np.float32)
    w[1, 5] = -3.0                       # single nonzero
    w[2, :] = -0.0                       # negative zeros
    w[3, 0], w[3, 1] = -2.0, 2.0         # +-absmax tie, element order in a byte
    codes, absmax = codec.quantize(w)
    q = codec.unpack_codes(codes, w.size).reshape(4, 64)
    assert absmax[0] == 0 and np.all(q[0] == 7) and np.all(codes[:32] == 0x77)
    assert absmax[1] == 3.0 and q[1, 5] == 0 and np.all(np.delete(q[1], 5) == 7)
    assert absmax[2] == 0 and np.all(q[2] == 7)
    assert q[3, 0] == 0 and q[3, 1] == 15 and codes[3 * 32] == 0x0F, "element 2i is the high nibble"


def test_exact_midpoint_tie_takes_lower_code():
    _, cb = codec.codebook()
    found = 0
    for k in range(15):
        mid = (float(cb[k]) + float(cb[k + 1])) / 2.0      # exact in binary64
        if float(np.float32(mid)) != mid:
            continue                                         # not representable: no tie possible
        w = np.zeros(64, np.float32)
        w[0] = 1.0
        w[1] = np.float32(mid)
        codes, _ = codec.quantize(w)
        assert codec.unpack_codes(codes, 64)[1] == k
        found += 1
    # plus the generic rule on values one ulp either side of every midpoint
    for k in range(15):
        mid = (float(cb[k]) + float(cb[k + 1])) / 2.0
        below = np.nextafter(np.float32(mid), np.float32(-2))
        above = np.nextafter(np.float32(mid), np.float32(2))
        if float(below) < mid:
            assert codec.nearest(float(below)) == k
        if float(above) > mid:
            assert codec.nearest(float(above)) == k + 1


@pytest.mark.parametrize("path", ["fp32", "bf16", "dq_bf16"])
def test_roundtrip_idempotence(path):
    w = synthetic.normal_f32((32, 1024), 0.02, 14)
    codes, absmax = codec.quantize(w)
    n = w.size
    if path == "fp32":
        back = codec.dequant_f32(codes, n, absmax=absmax)
    elif path == "bf16":
        back = codec.bf16_bits_to_f64(codec.dequant(codes, n, absmax=absmax)).astype(np.float32)
    else:
        qabs, scale, mu = codec.double_quant(absmax)
        back = codec.bf16_bits_to_f64(codec.dequant(codes, n, qabs=qabs, scale=scale, mu=mu)).astype(np.float32)
    codes2, _ = codec.quantize(back)
    assert np.array_equal(codes, codes2)


def test_codebook_points_roundtrip():
    # quantize o dequant is the identity on codebook points (per block, with
    # an end element fixing the absmax)
    _, cb = codec.codebook()
    w = np.tile(np.r_[cb, cb[::-1], cb, cb[::-1]].astype(np.float32), 3) * np.float32(0.5)
    codes, absmax = codec.quantize(w)
    assert np.all(absmax == 0.5)
    q = codec.unpack_codes(codes, w.size)
    assert np.array_equal(cb[q] * np.float32(0.5), w)


def test_rejects_empty_input():
    with pytest.raises(ValueError):
        codec.quantize(np.zeros(0, np.float32))


@pytest.mark.parametrize("n", [1, 2, 5, 63, 65, 127, 130, 1000, 4097])
def test_ragged_numel_equals_zero_padded_whole_blocks(n):
    """A partial last block: its absmax covers only the weights it has, and the
    bytes are those of W zero-padded to whole blocks (a zero weight gets code 7,
    and |0| never raises an absmax), cut to ceil(n/2) bytes."""
    w = synthetic.normal_f32((n,), 0.02, 100 + n)
    codes, absmax = codec.quantize(w)
    pad = np.zeros(-(-n // 64) * 64, np.float32)
    pad[:n] = w
    cp, ap = codec.quantize(pad)
    assert codes.size == (n + 1) // 2 and absmax.size == -(-n // 64)
    assert np.array_equal(codes, cp[:(n + 1) // 2])
    assert np.array_equal(absmax, ap)
    if n % 2:
        assert codes[-1] & 15 == 7
    # dequant of the ragged codes: the first n weights of the padded dequant
    assert np.array_equal(codec.dequant(codes, n, absmax=absmax), codec.dequant(cp, pad.size, absmax=ap)[:n])


def test_ragged_block_brute_force():
    """Five weights, worked by hand in binary64: nearest book entry of
    fp32(w / max|w|), lower code on ties, and the odd-numel padding nibble."""
    w = np.array([0.3, -0.05, 0.012, -0.6, 0.2], np.float32)
    codes, absmax = codec.quantize(w)
    assert absmax[0] == np.float32(0.6)
    cb = codec.cb32().astype(np.float64)
    q = []
    for v in w:
        x = float(np.float32(v) / np.float32(0.6))
        d = [abs(x - c) for c in cb]
        q.append(min(range(16), key=lambda k: (d[k], k)))
    assert q[3] == 0  # -absmax is the bottom of the book
    expect = [(q[0] << 4) | q[1], (q[2] << 4) | q[3], (q[4] << 4) | 7]
    assert list(codes) == expect


def test_sixteen_bit_widening_is_exact():
    """bf16 and fp16 weights enter the quantizer as their exact fp32 values:
    checked against torch's bfloat16 and NumPy's float16 conversions on every
    16-bit pattern, and on hand-picked values."""
    import torch
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = codec.widen16(bits, "f16")
    ref = bits.view(np.float16).astype(np.float32)
    same = (f.view(np.uint32) == ref.view(np.uint32)) | (np.isnan(f) & np.isnan(ref))
    assert same.all()
    b = codec.widen16(bits, "bf16")
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    same = (b.view(np.uint32) == t.view(np.uint32)) | (np.isnan(b) & np.isnan(t))
    assert same.all()
    assert codec.widen16(np.array([0x0001], np.uint16), "f16")[0] == np.float32(2.0 ** -24)
    assert codec.widen16(np.array([0x3C00, 0xC000], np.uint16), "f16").tolist() == [1.0, -2.0]
    assert codec.widen16(np.array([0x3F80, 0xBF00], np.uint16), "bf16").tolist() == [1.0, -0.5]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
def test_quantize16_is_quantize_of_the_widened_weights(kind):
    g = np.random.Generator(np.random.PCG64(5))
    w = (g.standard_normal(1000) * 0.02).astype(np.float32)
    bits = (w.view(np.uint32) >> 16).astype(np.uint16) if kind == "bf16" else w.astype(np.float16).view(np.uint16)
    codes, absmax = codec.quantize16(bits, kind)
    c2, a2 = codec.quantize(codec.widen16(bits, kind))
    assert np.array_equal(codes, c2) and np.array_equal(absmax, a2)

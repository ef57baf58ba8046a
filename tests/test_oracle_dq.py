"""Pins of the oracle's double quantization and doubleDequant.

Sources: "LoRA 与 QLoRA", QLoRA section 2 (r_j = (a_j - mu)/b, 8-bit rhat_j,
ahat_j = mu + b rhat_j, about 4.127 bit/param); deck "3 QLoRA Finetuning",
card 4 (8/64 + 32/(64*256) ~ 0.127 bits, blocks of 256); jjjymmm.cn 2024/03
QLoRA post, "Double Quantization" (the same count, saving 0.373) and "QLoRA"
(doubleDequant: constants first, then weights); deck card 1 (BF16 compute).
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from bit_nf4_quantized_07_b200 import synthetic
from oracle import codec
from tests.conftest import read_golden_values


def _printed():
    out = {}
    for line in read_golden_values("dq_storage_printed.txt"):
        k, v = line.split()[:2]
        out[k] = float(v)
    return out


def test_bits_per_param_closed_forms_against_actual_byte_counts():
    p = _printed()
    numel = 4096 * 4096
    w = synthetic.normal_f32((numel // 64, 64), 0.02, 21)
    codes, absmax = codec.quantize(w)
    qabs, scale, mu = codec.double_quant(absmax)
    plain_bits = 8.0 * absmax.nbytes / numel
    dq_bytes = qabs.nbytes + scale.nbytes + np.float32(mu).nbytes
    dq_bits = 8.0 * dq_bytes / numel
    assert dq_bytes == codec.constant_bytes(numel)
    assert plain_bits == p["plain_constant_bits"]
    assert 8.0 * codes.nbytes / numel + plain_bits == p["plain_total_bits"]
    # per-tensor mean mu is the only term not in the printed count
    assert dq_bits - 32.0 / numel == 8 / 64 + 32 / (64 * 256)
    assert round(dq_bits, 3) == p["dq_constant_bits"]
    assert round(plain_bits - dq_bits, 3) == p["dq_saving_bits"]
    assert round(plain_bits - dq_bits, 2) == p["dq_saving_bits_card"]
    assert round(8.0 * codes.nbytes / numel + dq_bits, 3) == p["dq_total_bits"]
    saving_gb = 65e9 * (plain_bits - dq_bits) / 8 / 1e9
    assert round(saving_gb) == p["saving_65b_gb"]


def test_mean_is_the_nearest_binary32_to_the_exact_mean():
    """mu is the mean of the block constants kept in 32 bits: the binary32
    value nearest to the exact rational mean, ties to even.  Checked against
    an independent exact sum (Python fractions of every value) and a rounding
    of that rational by bisection over the binary32 grid."""
    def nearest_by_search(x: Fraction) -> np.float32:
        f = np.float32(float(x))  # within one ulp of x
        best = None
        for cand in (np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))):
            d = abs(Fraction(float(cand)) - x)
            key = (d, int(np.array([cand], np.float32).view(np.uint32)[0]) & 1)
            if best is None or key < best[0]:
                best = (key, cand)
        return best[1]
    for seed, nb in ((31, 4096), (32, 1000), (33, 1), (34, 70001), (36, 3)):
        a = np.abs(synthetic.normal_f32(nb, 0.02, seed))
        exact = sum((Fraction(float(x)) for x in a), Fraction(0)) / nb
        assert codec.dq_mean(a) == nearest_by_search(exact)


def test_mean_closed_forms_and_ties():
    f32 = np.float32
    u = 2.0 ** -23
    cases = [
        ([0.25] * 5, 0.25),                              # a constant
        ([1.0, 1.0 + u], 1.0),                           # exact midpoint, even neighbour below
        ([1.0 + u, 1.0 + 2 * u], 1.0 + 2 * u),           # exact midpoint, even neighbour above
        ([2.0 ** -149, 0.0], 0.0),                       # half of the smallest subnormal: tie to 0
        ([2.0 ** -149, 2.0 ** -149, 0.0], 2.0 ** -149),  # two thirds of it: rounds up
        ([-1.0, 3.0], 1.0),                              # signs
        ([float(np.finfo(np.float32).max)] * 2, float(np.finfo(np.float32).max)),  # the exact sum overflows fp32
        ([0.1] * 1000, float(f32(0.1))),                 # a repeated binary32 value
    ]
    for vals, want in cases:
        assert codec.dq_mean(np.array(vals, f32)) == f32(want), vals


def test_binary32_rounding_of_exact_rationals_matches_numpy_casts():
    """nearest_f32 rounds an exact rational; for rationals that are binary64
    values, numpy's float64 -> float32 cast is that correct rounding."""
    rng = np.random.Generator(np.random.PCG64(37))
    x = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-40, 38, 2000),
                        rng.standard_normal(200) * 2.0 ** -140,  # subnormal range
                        (np.float32(rng.standard_normal(200)).astype(np.float64) +
                         np.spacing(np.float32(1.0)) / 2)])      # near binary32 midpoints
    for v in x:
        fr = Fraction(float(v)) * 2 ** 149
        got = codec.nearest_f32(fr.numerator, fr.denominator)
        assert got == np.float32(v), v


def test_dq_error_bound_extremes_and_range():
    w = synthetic.normal_f32((1000 * 64 // 64, 64 * 64), 0.02, 36)  # 64 000 blocks, last group partial
    _, absmax = codec.quantize(w)
    nb = absmax.size
    qabs, scale, mu = codec.double_quant(absmax)
    assert scale.size == (nb + 255) // 256
    assert qabs.min() >= -127 and qabs.max() <= 127
    ahat = codec.dq_restore(qabs, scale, mu)
    b = np.repeat(scale, 256)[:nb].astype(np.float64)
    err = np.abs(ahat.astype(np.float64) - absmax.astype(np.float64))
    ulp = np.spacing(np.abs(absmax)).astype(np.float64)
    assert np.all(err <= b / 2 + 2 * ulp + np.spacing(np.float32(mu)))
    for g in range(scale.size):
        blk = qabs[g * 256:(g + 1) * 256]
        assert np.max(np.abs(blk.astype(np.int32))) == 127, "the group's extreme maps to +-127"


def test_dq_degenerate_groups():
    a = np.full(512, 0.25, np.float32)              # all equal: b == 0
    qabs, scale, mu = codec.double_quant(a)
    assert mu == np.float32(0.25) and np.all(scale == 0) and np.all(qabs == 0)
    assert np.all(codec.dq_restore(qabs, scale, mu) == np.float32(0.25))
    a = np.zeros(300, np.float32)                    # all-zero weights -> zero constants
    qabs, scale, mu = codec.double_quant(a)
    assert mu == 0 and np.all(qabs == 0)


def test_int8_dq_rint_ties_worked_by_hand():
    """A group whose quotients are exact halves ("LoRA 与 QLoRA" section 2:
    r_j = (a_j - mu) / b rounded to 8 bits), worked by hand.  The constants are
    mu +- {127, 2.5, 3.5, 0.5, 1.5} with mu = 200: the exact mean is 200, so
    d_j = a_j - 200 exactly, max|d| = 127 gives b = 127 / 127 = 1 exactly, and
    r_j = d_j.  Ties go to the even integer: 2.5 -> 2, 3.5 -> 4, 0.5 -> 0,
    1.5 -> 2 (and the negatives likewise).  Rounding half away from zero
    (3, 4, 1, 2) or truncation (2, 3, 0, 1) fails here."""
    d = np.array([127, -127, 2.5, -2.5, 3.5, -3.5, 0.5, -0.5, 1.5, -1.5], np.float64)
    a = (200.0 + d).astype(np.float32)
    assert np.array_equal(a.astype(np.float64) - 200.0, d)       # the constants are exact
    qabs, scale, mu = codec.double_quant(a)
    assert mu == np.float32(200.0) and scale.tolist() == [1.0]
    assert qabs.tolist() == [127, -127, 2, -2, 4, -4, 0, 0, 2, -2]


def test_dq_restore_order_worked_by_hand():
    """ahat = mu + b rhat ("LoRA 与 QLoRA" section 2), in the written order:
    the product rounded to fp32 first, then the sum.  Worked by hand with
    b = 1 + 2^-23, rhat = 3, mu = -3: b rhat = 3 + 3 2^-23 lies halfway
    between the fp32 neighbours 3 + 2^-22 and 3 + 2^-21 (the spacing near 3 is
    2^-22) and rounds to the even one, 3 + 2^-21; adding mu = -3 is then exact,
    ahat = 2^-21.  A fused multiply-add rounds once, to 3 2^-23."""
    b = np.float32(1.0 + 2.0 ** -23)
    assert float(b) == 1.0 + 2.0 ** -23
    got = codec.dq_restore(np.array([3], np.int8), np.array([b], np.float32), np.float32(-3.0))
    assert float(got[0]) == 2.0 ** -21
    fma = float(np.float32(float(b) * 3.0 + (-3.0)))              # one rounding of the exact value
    assert fma == 3 * 2.0 ** -23 and fma != float(got[0])
    # and the doubleDequant of a block whose codes all hold the book's 1.0 (code 15)
    codes = np.full(32, 0xFF, np.uint8)
    bf = codec.dequant(codes, 64, qabs=np.array([3], np.int8), scale=np.array([b], np.float32), mu=np.float32(-3.0))
    assert np.all(bf == 0x3500)                                   # bf16 bits of 2^-21


def test_bf16_rounding_against_torch():
    g = np.random.Generator(np.random.PCG64(37))
    x = (g.standard_normal(200000) * 10.0 ** g.integers(-30, 30, 200000)).astype(np.float32)
    bits = x.view(np.uint32)
    bits[:1000] = (bits[:1000] & 0xFFFF0000) | 0x8000          # exact ties
    bits[1000:2000] = (bits[1000:2000] & 0xFFFF0000) | 0x7FFF
    ours = np.array([codec.bf16_rn(float(v)) for v in x], np.uint16)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_dequant_definition_and_special_codes():
    w = synthetic.normal_f32((64, 512), 0.02, 38)
    n = w.size
    codes, absmax = codec.quantize(w)
    qabs, scale, mu = codec.double_quant(absmax)
    q = codec.unpack_codes(codes, n).reshape(-1, 64)
    ahat = codec.dq_restore(qabs, scale, mu)
    f32 = codec.dequant_f32(codes, n, qabs=qabs, scale=scale, mu=mu).reshape(-1, 64)
    _, cb = codec.codebook()
    assert np.array_equal(f32, ahat[:, None] * cb[q])            # fp32 product, NumPy IEEE
    bf = codec.dequant(codes, n, qabs=qabs, scale=scale, mu=mu).reshape(-1, 64)
    ref = torch.from_numpy(np.ascontiguousarray(f32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf, ref)
    v = codec.bf16_bits_to_f64(bf)
    assert np.all(v[q == 7] == 0.0)
    top = codec.bf16_bits_to_f64(torch.from_numpy(ahat).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    tb = np.broadcast_to(top[:, None], q.shape)
    assert np.all(v[q == 15] == tb[q == 15]) and np.all(v[q == 0] == -tb[q == 0])
    # without DQ the plain absmax is the constant
    plain = codec.dequant_f32(codes, n, absmax=absmax).reshape(-1, 64)
    assert np.array_equal(plain, absmax[:, None] * cb[q])


# --- the "8-bit floats" reading of DQ (deck card 4): OCP FP8 E4M3 codes -----

def test_e4m3_decode_against_torch_and_the_format_definition():
    """Every code against torch.float8_e4m3fn's conversion (a library routine),
    plus values fixed by the format: 1.0, the largest 448, the smallest
    subnormal 2^-9, the smallest normal 2^-6, signed zero, the NaN codes."""
    vals = np.array([codec.e4m3_value(c) for c in range(256)])
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    both_nan = np.isnan(vals) & np.isnan(ref)
    assert np.all(both_nan | (vals == ref))
    assert vals[0x38] == 1.0 and vals[0x7E] == 448.0 and vals[0xFE] == -448.0
    assert vals[0x01] == 2.0 ** -9 and vals[0x08] == 2.0 ** -6 and vals[0x07] == 7 * 2.0 ** -9
    assert vals[0x00] == 0.0 and math.copysign(1.0, vals[0x80]) == -1.0
    assert np.isnan(vals[0x7F]) and np.isnan(vals[0xFF]) and np.isnan(vals).sum() == 2
    finite = vals[:0x7F]
    assert np.all(np.diff(finite) > 0), "non-negative codes increase with value"


def test_e4m3_encode_nearest_even_and_saturating():
    g = np.random.Generator(np.random.PCG64(17))
    x = np.concatenate([g.uniform(-448, 448, 4000), g.standard_normal(4000) * 0.01,
                        g.uniform(-2, 2, 4000)]).astype(np.float32)
    enc = np.array([codec.e4m3_encode(v) for v in x], np.uint8)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(enc, ref)
    # ties go to the even mantissa: 1.0625 lies halfway between 1.0 (0x38) and
    # 1.125 (0x39); 1.1875 halfway between 1.125 and 1.25 (0x3A)
    assert codec.e4m3_encode(1.0625) == 0x38 and codec.e4m3_encode(1.1875) == 0x3A
    assert codec.e4m3_encode(-1.0625) == 0xB8
    # halfway between the two smallest subnormals (2^-9 and 2^-8): to 2^-8 (code 2)
    assert codec.e4m3_encode(1.5 * 2.0 ** -9) == 0x02
    # beyond the largest finite value: saturate (no infinities in E4M3)
    for v, c in ((448.0, 0x7E), (460.0, 0x7E), (500.0, 0x7E), (1e30, 0x7E), (-1e30, 0xFE)):
        assert codec.e4m3_encode(v) == c


def test_e4m3_dq_group_extremes_error_bound_and_shared_mean():
    """Each group with b > 0 holds +-448 at its farthest constant; every
    restored constant is within half an E4M3 step of its true value (relative
    2^-4 in the normal range, 2^-10 absolute among subnormals) scaled by b,
    plus binary32 rounding; mu is the INT8 reading's mu."""
    a = np.abs(synthetic.normal_f32(256 * 40 + 77, 0.02, 23))
    q, b, mu = codec.double_quant(a, fmt="e4m3")
    q8, b8, mu8 = codec.double_quant(a, fmt="int8")
    assert np.float32(mu) == np.float32(mu8)
    assert q.dtype == np.uint8 and b.size == b8.size
    for g in range(b.size):
        grp = q[g * 256:(g + 1) * 256]
        assert b[g] > 0 and np.any((grp & 0x7F) == 0x7E)
    ah = codec.dq_restore(q, b, mu, fmt="e4m3").astype(np.float64)
    r = (a.astype(np.float64) - float(mu)) / np.repeat(b.astype(np.float64), 256)[:a.size]
    half_step = np.where(np.abs(r) >= 2.0 ** -6, np.abs(r) * 2.0 ** -4, 2.0 ** -10)
    bound = np.repeat(b.astype(np.float64), 256)[:a.size] * (half_step + 1e-6) + 2.0 ** -22 * np.abs(a)
    assert np.all(np.abs(ah - a) <= bound)


def test_e4m3_dq_degenerate_group_and_dequant_format():
    a = np.full(300, np.float32(0.25))                        # all equal -> b == 0 -> code 0
    q, b, mu = codec.double_quant(a, fmt="e4m3")
    assert np.all(q == 0) and np.all(b == 0) and mu == np.float32(0.25)
    # dequant reads the E4M3 codes through the same restore as dq_restore
    w = synthetic.normal_f32((64 * 600,), 0.02, 29)
    codes, absmax = codec.quantize(w)
    q, b, mu = codec.double_quant(absmax, fmt="e4m3")
    ah = codec.dq_restore(q, b, mu, fmt="e4m3")
    full = codec.dequant(codes, w.size, qabs=q, scale=b, mu=mu, fmt="e4m3")
    plain = codec.dequant(codes, w.size, absmax=ah)
    assert np.array_equal(full, plain)

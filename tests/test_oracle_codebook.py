"""Pins of the oracle's NF4 codebook against what the pages and mathematics fix.

Sources: jjjymmm.cn 2024/03 QLoRA post, "4-bit NormalFloat(NF4)" (the printed
quant book); "LoRA 与 QLoRA", QLoRA section 1 (quantiles, exact zero,
normalization to [-1, 1]); deck "3 QLoRA Finetuning", card 3 (separate negative
and positive halves sharing one zero).
"""
import math
from statistics import NormalDist

import numpy as np
import pytest
import scipy.special

from oracle import codec
from tests.conftest import read_golden_values

PRINTED = np.array([float(v) for v in read_golden_values("nf4_codebook_printed.txt")])


def test_quantile_matches_two_independent_library_routines():
    nd = NormalDist()
    for p in (0.5, 0.51, 0.6, 0.75, 0.9, 0.95, codec.DELTA, 0.99, 0.999, 1e-6, 0.02):
        q = codec.normal_quantile(p)
        assert abs(q - nd.inv_cdf(p)) <= 1e-12 * max(1.0, abs(q))
        assert abs(q - scipy.special.ndtri(p)) <= 1e-12 * max(1.0, abs(q))
        assert abs(codec.normal_cdf(q) - p) <= 1e-15


def test_codebook_structure():
    c64, c32 = codec.codebook()
    assert c32.dtype == np.float32 and c32.size == 16
    assert np.all(np.diff(c32.astype(np.float64)) > 0), "ascending and distinct"
    assert c32[7] == 0.0 and not np.signbit(c32[7]), "exact zero (0 -> 0)"
    assert c32[0] == -1.0 and c32[15] == 1.0, "normalized ends are exactly -1, +1"
    assert np.sum(c32 < 0) == 7 and np.sum(c32 > 0) == 8, "asymmetric halves, all 16 codes used"
    assert np.all(c32 == c64.astype(np.float32))


def test_codebook_matches_printed_table():
    _, c32 = codec.codebook()
    dev = np.abs(c32.astype(np.float64) - PRINTED)
    # 4-decimal printing: within half a unit of the 4th decimal.  The printed
    # -0.0911 sits on the rounding boundary of -0.09105, hence 5.1e-5.
    assert dev.max() <= 5.1e-5, dev
    assert np.all(np.delete(dev, 6) < 5.0e-5)
    assert dev[6] > 5.0e-5          # -0.09105 printed as -0.0911: on the boundary


def test_offset_window_is_pinned_by_the_printed_table():
    def maxdev(delta):
        c64, _ = codec.codebook(delta)
        return np.max(np.abs(c64 - PRINTED))

    for d in (0.96768, codec.DELTA, 0.96773):
        assert maxdev(d) <= 1.0e-4
    for d in (0.9670, 0.9650, 0.9685, 0.975, 0.96):
        assert maxdev(d) > 1.0e-4


def test_codebook_recomputed_with_scipy_gives_same_fp32_bits():
    d = codec.DELTA
    pos = [scipy.special.ndtri(d + i * (0.5 - d) / 8.0) for i in range(8)]
    neg = [-scipy.special.ndtri(d + i * (0.5 - d) / 7.0) for i in range(7)]
    top = scipy.special.ndtri(d)
    v = np.sort(np.array(pos + neg + [0.0]) / top).astype(np.float32)
    _, c32 = codec.codebook()
    assert np.array_equal(v.view(np.uint32), c32.view(np.uint32))


def test_symmetric_endpoint_formula_is_not_the_table():
    # "LoRA 与 QLoRA" prints q_i = (Q(i/17) + Q((i+1)/17)) / 2 and asks how the
    # endpoints are handled.  Taken over i = 1..15 and normalized it gives a
    # symmetric 15-value grid, unlike the asymmetric printed table: the table
    # is the separate-halves construction, not this formula.
    q = np.array([0.5 * (codec.normal_quantile(i / 17) + codec.normal_quantile((i + 1) / 17))
                  for i in range(1, 16)])
    q = q / np.max(np.abs(q))
    assert np.allclose(q, -q[::-1], atol=1e-12)
    assert not np.allclose(PRINTED, -PRINTED[::-1], atol=1e-3)
    assert abs(np.min(q[q > 1e-9]) - 0.0796) > 0.02


def test_minimum_gap():
    _, c32 = codec.codebook()
    gaps = np.diff(c32.astype(np.float64))
    assert math.isclose(gaps.min(), 0.0796, abs_tol=1e-4)
    assert gaps.argmin() == 7   # between 0 and the first positive value

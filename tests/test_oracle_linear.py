"""Pins of the float64 forward/backward oracle.

Sources: "LoRA 与 QLoRA", section LoRA (Delta W = s B A, y = W0 x + s B(Ax),
only A and B trained) and "rank 的证明" (rank(BA) <= r); deck
"3 QLoRA Finetuning", card 1 (gradients flow through the dequantized weights).
"""
import numpy as np
import pytest
import torch

from oracle import linear


def _rand(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


def _problem(dout=24, din=40, n=5, r=3, s=1.7, seed=0):
    return (_rand((dout, din), seed + 1, 0.1), _rand((n, din), seed + 2), _rand((r, din), seed + 3, 0.3),
            _rand((dout, r), seed + 4, 0.3), s, _rand((n, dout), seed + 5))


def test_backward_matches_central_finite_differences():
    Wp, X, A, B, s, dY = _problem()
    dX, dA, dB = linear.backward(Wp, X, A, B, s, dY)

    def loss(Wp_, X_, A_, B_):
        return float(np.sum(dY * linear.forward(Wp_, X_, A_, B_, s)[0]))

    h = 1e-4
    for name, T, G in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        num = np.zeros_like(T)
        for idx in np.ndindex(T.shape):
            Tp, Tm = T.copy(), T.copy()
            Tp[idx] += h
            Tm[idx] -= h
            args = {"X": (Wp, X, A, B), "A": (Wp, X, A, B), "B": (Wp, X, A, B)}[name]
            ap = list(args)
            am = list(args)
            pos = {"X": 1, "A": 2, "B": 3}[name]
            ap[pos], am[pos] = Tp, Tm
            num[idx] = (loss(*ap) - loss(*am)) / (2 * h)
        assert np.allclose(num, G, rtol=1e-7, atol=1e-8), name


def test_forward_equals_merged_weight_form():
    Wp, X, A, B, s, _ = _problem(dout=33, din=64, n=7, r=5, s=2.0, seed=10)
    Y, U = linear.forward(Wp, X, A, B, s)
    assert Y.shape == (7, 33) and U.shape == (7, 5)
    assert np.allclose(Y, linear.merged_forward(Wp, X, A, B, s), rtol=1e-12, atol=1e-12)


def test_special_cases_reduce_to_textbook_gemm():
    Wp, X, A, B, s, dY = _problem(seed=20)
    ref = torch.matmul(torch.from_numpy(X), torch.from_numpy(Wp).T).numpy()
    assert np.allclose(linear.forward(Wp, X, A, np.zeros_like(B), s)[0], ref, rtol=1e-13, atol=1e-13)
    assert np.allclose(linear.forward(Wp, X, A, B, 0.0)[0], ref, rtol=1e-13, atol=1e-13)
    dX, dA, dB = linear.backward(Wp, X, A, B, 0.0, dY)
    assert np.allclose(dX, torch.matmul(torch.from_numpy(dY), torch.from_numpy(Wp)).numpy())
    assert np.all(dA == 0) and np.all(dB == 0)
    # all-zero frozen weight: only the adapter path remains
    Y0, U = linear.forward(np.zeros_like(Wp), X, A, B, s)
    assert np.allclose(Y0, s * torch.matmul(torch.from_numpy(U), torch.from_numpy(B).T).numpy())


def test_linearity_in_s():
    Wp, X, A, B, _, dY = _problem(seed=30)
    Y0 = linear.forward(Wp, X, A, B, 0.0)[0]
    Y1 = linear.forward(Wp, X, A, B, 1.0)[0]
    Y3 = linear.forward(Wp, X, A, B, 3.0)[0]
    assert np.allclose(Y3 - Y0, 3.0 * (Y1 - Y0), rtol=1e-12, atol=1e-12)
    _, dA1, dB1 = linear.backward(Wp, X, A, B, 1.0, dY)
    _, dA3, dB3 = linear.backward(Wp, X, A, B, 3.0, dY)
    assert np.allclose(dA3, 3 * dA1) and np.allclose(dB3, 3 * dB1)


@pytest.mark.parametrize("r", [1, 2, 8, 16])
def test_rank_of_update_bounded_by_r(r):
    B = _rand((96, r), 40 + r)
    A = _rand((r, 80), 50 + r)
    assert np.linalg.matrix_rank(B @ A) <= r
    assert np.linalg.matrix_rank(B @ A) == r        # generic factors reach it


def test_error_metrics():
    T = np.array([[1.0, -2.0], [0.5, 4.0]])
    assert linear.normwise_error(T, T) == 0.0
    assert linear.normwise_error(T + 0.04, T) == pytest.approx(0.01)
    assert linear.frobenius_error(2 * T, T) == pytest.approx(1.0)

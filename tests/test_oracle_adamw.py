"""Pins of the AdamW oracle (the paged optimizer's update rule).

Sources: deck "3 QLoRA Finetuning" card 5 (paged optimizers), "LoRA 与 QLoRA"
QLoRA usage notes (paged_adamw_32bit); the update itself is the published
AdamW (Loshchilov & Hutter, ICLR 2019), which the pages do not write out.
"""
import numpy as np
import pytest
import torch

from oracle import adamw


@pytest.mark.parametrize("wd", [0.0, 0.01, 0.1])
def test_matches_torch_adamw_over_several_steps(wd):
    """torch.optim.AdamW (a library routine) in float64 on the same data."""
    g = np.random.Generator(np.random.PCG64(3))
    n, steps, lr, b1, b2, eps = 1000, 7, 3e-3, 0.9, 0.995, 1e-8
    p0 = g.standard_normal(n) * 0.05
    grads = [g.standard_normal(n) * 10 ** g.uniform(-6, 0) for _ in range(steps)]
    tp = torch.nn.Parameter(torch.from_numpy(p0.copy()))
    opt = torch.optim.AdamW([tp], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd)
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    for t in range(1, steps + 1):
        tp.grad = torch.from_numpy(grads[t - 1].copy())
        opt.step()
        p, m, v = adamw.adamw_step(p, grads[t - 1], m, v, t, lr, b1, b2, eps, wd)
        st = opt.state[tp]
        np.testing.assert_allclose(p, tp.detach().numpy(), rtol=1e-13, atol=1e-16)
        np.testing.assert_allclose(m, st["exp_avg"].numpy(), rtol=1e-13, atol=0)
        np.testing.assert_allclose(v, st["exp_avg_sq"].numpy(), rtol=1e-13, atol=0)


def test_first_step_moves_each_weight_by_lr_times_sign():
    """t = 1 from zero states: m_hat = g and v_hat = g^2 exactly, so the step is
    lr g / (|g| + eps), i.e. lr sign(g) up to eps."""
    g = np.array([3.0, -0.5, 1e-3, -2e-2])
    p, m, v = adamw.adamw_step(np.zeros(4), g, np.zeros(4), np.zeros(4), 1, 0.01, eps=1e-8)
    np.testing.assert_allclose(p, -0.01 * g / (np.abs(g) + 1e-8), rtol=1e-14)
    np.testing.assert_allclose(m, 0.1 * g, rtol=1e-13)
    np.testing.assert_allclose(v, 0.001 * g * g, rtol=1e-13)  # 1 - 0.999 is not exactly 0.001 in binary64


def test_constant_gradient_keeps_unit_steps_and_decay_shrinks():
    """A constant gradient g for t steps gives m_hat = g and v_hat = g^2 at every
    step (the bias corrections undo the zero start), so each step moves the
    weight by lr g / (|g| + eps); weight decay alone multiplies by (1 - lr wd)."""
    g = np.array([0.7, -1.3])
    p, m, v = np.array([1.0, 2.0]), np.zeros(2), np.zeros(2)
    for t in range(1, 6):
        p_prev = p
        p, m, v = adamw.adamw_step(p, g, m, v, t, 0.05)
        np.testing.assert_allclose(p_prev - p, 0.05 * g / (np.abs(g) + 1e-8), rtol=1e-12)
    p, _, _ = adamw.adamw_step(np.array([2.0]), np.array([0.0]), np.zeros(1), np.zeros(1), 1, 0.1, wd=0.5)
    assert p[0] == pytest.approx(2.0 * (1 - 0.1 * 0.5), rel=1e-15)

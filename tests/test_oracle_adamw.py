"""Pins of the AdamW oracle (oracle/adamw.py): against torch.optim.AdamW run
on the CPU in float64 (a library implementation that shares no code with the
oracle), against the closed form of the first step (m_hat = g and
v_hat = g^2, so the step is lr g / (|g| + eps) plus the decay), and against
the limits the algorithm fixes (no gradient and no decay: nothing moves;
b1 = b2 = 0: every step is a sign step of size lr)."""
import numpy as np
import pytest
import torch

from oracle.adamw import adamw_step


@pytest.mark.parametrize("lr,b1,b2,eps,wd", [(1e-3, 0.9, 0.999, 1e-8, 0.0), (2e-2, 0.8, 0.95, 1e-6, 0.1),
                                             (5e-4, 0.0, 0.5, 1e-3, 0.01)])
def test_matches_torch_adamw_float64(lr, b1, b2, eps, wd):
    rng = np.random.default_rng(1)
    p0 = rng.normal(0, 0.05, 257)
    grads = [rng.normal(0, 1e-2, 257) for _ in range(6)]
    tp = torch.tensor(p0, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([tp], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd, foreach=False)
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    for t, g in enumerate(grads, start=1):
        tp.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        p, m, v = adamw_step(p, m, v, g, t, lr, b1, b2, eps, wd)
        np.testing.assert_allclose(p, tp.detach().numpy(), rtol=1e-13, atol=1e-15)
    st = opt.state[tp]
    np.testing.assert_allclose(m, st["exp_avg"].numpy(), rtol=1e-13, atol=1e-18)
    np.testing.assert_allclose(v, st["exp_avg_sq"].numpy(), rtol=1e-13, atol=1e-20)


def test_first_step_closed_form():
    rng = np.random.default_rng(2)
    p0, g = rng.normal(0, 0.05, 100), rng.normal(0, 1e-3, 100)
    lr, eps, wd = 1e-2, 1e-8, 0.05
    p, m, v = adamw_step(p0, 0 * p0, 0 * p0, g, 1, lr, 0.9, 0.999, eps, wd)
    np.testing.assert_allclose(p, p0 * (1 - lr * wd) - lr * g / (np.abs(g) + eps), rtol=1e-12)
    np.testing.assert_allclose(m, 0.1 * g, rtol=1e-12)
    np.testing.assert_allclose(v, 0.001 * g * g, rtol=1e-12)


def test_limits():
    rng = np.random.default_rng(3)
    p0 = rng.normal(0, 0.05, 64)
    z = np.zeros_like(p0)
    p, m, v = adamw_step(p0, z, z, z, 3, 1e-2, 0.9, 0.999, 1e-8, 0.0)
    assert np.array_equal(p, p0) and not m.any() and not v.any()
    g = rng.normal(0, 1.0, 64)
    p, _, _ = adamw_step(p0, z, z, g, 5, 1e-2, 0.0, 0.0, 1e-12, 0.0)
    np.testing.assert_allclose(p, p0 - 1e-2 * np.sign(g), rtol=1e-9)

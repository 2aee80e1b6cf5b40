"""Pins for the AdamW oracle (CPU): the closed forms of the first step and of
a constant gradient (bias correction makes both exact), pure decoupled weight
decay, and PyTorch's own AdamW (an independent implementation) over several
steps with weight decay and a gradient scale."""
import numpy as np
import torch

from oracle.optim import adamw_step

B1, B2, EPS = 0.9, 0.999, 1e-8


def _grads(n=257, seed=0):
    g = np.random.default_rng(seed).standard_normal(n)
    g[:8] = [1e-9, -1e-9, 1e-8, -3e-8, 0.0, 5.0, -2e-3, 1e-7]  # near eps: pins where eps enters
    return g


def test_first_step_closed_form():
    # from zero moments, m_hat = g and v_hat = g^2 exactly: theta moves by lr g / (|g| + eps)
    g = _grads()
    th0 = np.random.default_rng(1).standard_normal(g.size)
    lr = 5e-4
    th, m, v = adamw_step(th0, g, np.zeros_like(g), np.zeros_like(g), 1, lr, B1, B2, EPS)
    np.testing.assert_allclose(th, th0 - lr * g / (np.abs(g) + EPS), rtol=1e-13, atol=1e-18)
    np.testing.assert_allclose(m, (1 - B1) * g, rtol=1e-15, atol=0)
    np.testing.assert_allclose(v, (1 - B2) * g * g, rtol=1e-15, atol=0)


def test_constant_gradient_closed_form():
    # m_t = (1 - beta1^t) g and v_t = (1 - beta2^t) g^2, so every step moves theta by lr g / (|g| + eps)
    g = _grads(seed=2)
    th0 = np.random.default_rng(3).standard_normal(g.size)
    th, m, v = th0.copy(), np.zeros_like(g), np.zeros_like(g)
    lr = 1e-2
    for t in range(1, 7):
        th, m, v = adamw_step(th, g, m, v, t, lr, B1, B2, EPS)
        np.testing.assert_allclose(m, (1 - B1 ** t) * g, rtol=1e-13, atol=0)
        np.testing.assert_allclose(v, (1 - B2 ** t) * g * g, rtol=1e-12, atol=0)
        np.testing.assert_allclose(th, th0 - t * lr * g / (np.abs(g) + EPS), rtol=1e-12, atol=1e-15)


def test_pure_decoupled_weight_decay():
    # zero gradient: the moments stay zero and theta shrinks geometrically by (1 - lr wd)
    th0 = np.random.default_rng(4).standard_normal(64)
    th, m, v = th0.copy(), np.zeros(64), np.zeros(64)
    lr, wd = 1e-2, 0.1
    for t in range(1, 5):
        th, m, v = adamw_step(th, np.zeros(64), m, v, t, lr, B1, B2, EPS, weight_decay=wd)
        assert not m.any() and not v.any()
        np.testing.assert_allclose(th, th0 * (1 - lr * wd) ** t, rtol=1e-14, atol=0)


def test_matches_torch_adamw():
    # several steps with fresh gradients, weight decay and a gradient scale
    rng = np.random.default_rng(5)
    n, lr, wd, scale = 300, 3e-2, 0.1, 0.25
    th0 = rng.standard_normal(n)
    p = torch.tensor(th0, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([p], lr=lr, betas=(B1, B2), eps=EPS, weight_decay=wd, foreach=False)
    th, m, v = th0.copy(), np.zeros(n), np.zeros(n)
    for t in range(1, 6):
        g = rng.standard_normal(n) * (10.0 ** rng.integers(-6, 1, n))
        p.grad = torch.tensor(g * scale, dtype=torch.float64)
        opt.step()
        th, m, v = adamw_step(th, g, m, v, t, lr, B1, B2, EPS, weight_decay=wd, grad_scale=scale)
        st = opt.state[p]
        np.testing.assert_allclose(th, p.detach().numpy(), rtol=1e-13, atol=1e-16)
        # PyTorch forms m as a lerp (another rounding order): a few fp64 ulps apart
        np.testing.assert_allclose(m, st["exp_avg"].numpy(), rtol=1e-12, atol=0)
        np.testing.assert_allclose(v, st["exp_avg_sq"].numpy(), rtol=1e-12, atol=0)


def test_step_index_starts_at_one():
    try:
        adamw_step(np.zeros(2), np.zeros(2), np.zeros(2), np.zeros(2), 0, 1e-3)
    except ValueError:
        return
    raise AssertionError("t = 0 must be refused")

"""Pins for the LoRA linear oracle (CPU): central finite differences, the
B = 0 and adapters-off special cases, and the merged-weight closed form."""
import numpy as np

from oracle.lora import lora_bwd, lora_fwd


def _setup(T=5, n_in=16, n_out=12, r=2, seed=0):
    g = np.random.default_rng(seed)
    return (g.standard_normal((T, n_in)), g.standard_normal((n_out, n_in)) * 0.3,
            g.standard_normal((r, n_in)) * 0.3, g.standard_normal((n_out, r)) * 0.3,
            g.standard_normal((T, n_out)))


def test_finite_differences():
    x, W, A, B, R = _setup()
    s = 2.0
    L = lambda x_, A_, B_: float(np.sum(lora_fwd(x_, W, A_, B_, s)[0] * R))
    dx, dA, dB = lora_bwd(x, W, A, B, s, R)
    h = 1e-6
    for arr, grad, name in ((x, dx, "x"), (A, dA, "A"), (B, dB, "B")):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            p, m = arr.copy(), arr.copy()
            p[idx] += h
            m[idx] -= h
            args = {"x": (x, A, B), "A": (x, A, B), "B": (x, A, B)}[name]
            lp = L(*[p if a is arr else a for a in args])
            lm = L(*[m if a is arr else a for a in args])
            num[idx] = (lp - lm) / (2 * h)
        rel = np.linalg.norm(num - grad) / np.linalg.norm(grad)
        assert rel < 1e-6, (name, rel)


def test_B_zero_reproduces_base_exactly():
    x, W, A, B, R = _setup()
    y, _ = lora_fwd(x, W, A, np.zeros_like(B), 2.0)
    assert np.array_equal(y, x @ W.T)


def test_adapters_off_is_base_model():
    x, W, A, B, R = _setup()
    y, _ = lora_fwd(x, W, A, B, 2.0, adapters_on=False)
    assert np.array_equal(y, x @ W.T)
    dx, dA, dB = lora_bwd(x, W, A, B, 2.0, R, adapters_on=False)
    assert np.array_equal(dx, R @ W) and not dA.any() and not dB.any()


def test_merged_weight_closed_form():
    """LoRA is a rank-r update of the frozen weight: y = x (W + s B A)^T."""
    x, W, A, B, R = _setup(T=7, n_in=32, n_out=24, r=4, seed=3)
    y, u = lora_fwd(x, W, A, B, 0.5)
    np.testing.assert_allclose(y, x @ (W + 0.5 * B @ A).T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(u, x @ A.T, rtol=1e-12, atol=1e-12)
    # and the gradient w.r.t. x is the transpose of the same merged map
    dx, _, _ = lora_bwd(x, W, A, B, 0.5, R)
    np.testing.assert_allclose(dx, R @ (W + 0.5 * B @ A), rtol=1e-12, atol=1e-12)

"""The AdamW kernel (soup_adamw_step) against the AdamW oracle.

Every step is compared with the oracle fed the kernel's own fp32 state from
the step before (theta, m, v) and the same fp32 gradients, with the
hyperparameters as the fp32 values the C ABI receives.  Tolerances follow the
kernel's fp32 arithmetic (u = 2^-24 per rounding; m and v take at most 4
and 6 roundings of terms bounded by the magnitudes below, the update about 18
relative to its magnitude; the bounds leave margin over those counts):
  m:     8u (beta1 |m_old| + (1 - beta1) |g|)
  v:     8u (beta2 v_old + (1 - beta2) g^2)
  theta: 32u * step_size * (beta1 |m_old| + (1 - beta1) |g|) / denom + 4u (|theta_old| + |theta_new|)
where g is the scaled gradient and denom = sqrt(v_hat) + eps.  The bf16
working copy must be the round-to-nearest-even of the kernel's own new fp32
theta, bit for bit, and a cleared gradient must be exactly zero."""
import numpy as np
import pytest
import torch

from oracle.nf4 import round_to_bf16
from oracle.optim import adamw_step

pytestmark = pytest.mark.gpu
L = None
U = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _mods():
    global L
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from layer_streamed_qlora_b200 import _lib
    _lib.lib()
    L = _lib
    yield
    assert _lib.device_error() == 0


def f32(x):
    return float(np.float32(x))


def _grads(rng, n):
    # magnitudes over six decades, so that eps and the moment mix both matter
    return (rng.standard_normal(n) * 10.0 ** rng.integers(-6, 1, n)).astype(np.float32)


def _check_step(theta0, g, m0, v0, t, hp, theta, m, v, idx=None):
    """theta0, g, m0, v0: the kernel's inputs (fp32 numpy); theta, m, v: its outputs."""
    lr, b1, b2, eps, wd, gs = (f32(hp[k]) for k in ("lr", "beta1", "beta2", "eps", "weight_decay", "grad_scale"))
    if idx is not None:
        theta0, g, m0, v0, theta, m, v = (a[idx] for a in (theta0, g, m0, v0, theta, m, v))
    th_r, m_r, v_r = adamw_step(theta0.astype(np.float64), g.astype(np.float64), m0.astype(np.float64),
                                v0.astype(np.float64), t, lr, b1, b2, eps, wd, gs)
    ga = np.abs(g.astype(np.float64) * gs)
    mag_m = b1 * np.abs(m0.astype(np.float64)) + (1 - b1) * ga
    mag_v = b2 * v0.astype(np.float64) + (1 - b2) * ga * ga
    assert np.all(np.abs(m - m_r) <= 8 * U * mag_m), float(np.max(np.abs(m - m_r) / np.maximum(mag_m, 1e-300)))
    assert np.all(np.abs(v - v_r) <= 8 * U * mag_v), float(np.max(np.abs(v - v_r) / np.maximum(mag_v, 1e-300)))
    denom = np.sqrt(v_r / (1 - b2 ** t)) + eps
    step = lr / (1 - b1 ** t)
    tol = 32 * U * step * mag_m / denom + 4 * U * (np.abs(theta0.astype(np.float64)) + np.abs(th_r))
    err = np.abs(theta.astype(np.float64) - th_r)
    assert np.all(err <= tol), float(np.max(err / np.maximum(tol, 1e-300)))


def _dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dtype)


@pytest.mark.parametrize("n", [1, 3, 4, 1027, 148 * 8 * 256 * 4 * 2 + 5])
@pytest.mark.parametrize("wd,gs", [(0.0, 1.0), (0.1, 0.25)])
def test_adamw_matches_oracle_over_steps(n, wd, gs):
    # ragged sizes (scalar tail, one vector group, several grid-stride rounds + tail)
    rng = np.random.default_rng(n + int(wd * 10))
    hp = dict(lr=3e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=wd, grad_scale=gs)
    theta = _dev((rng.standard_normal(n) * 0.02).astype(np.float32))
    bf = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    m = torch.zeros(n, device="cuda")
    v = torch.zeros(n, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in range(1, 4):
        g_host = _grads(rng, n)
        grad = _dev(g_host)
        th0, m0, v0 = theta.cpu().numpy(), m.cpu().numpy(), v.cpu().numpy()
        L.soup_adamw_step(theta, bf, grad, m, v, hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], wd, gs, t,
                          zero_grad=True, nonfinite=flag)
        torch.cuda.synchronize()
        th1 = theta.cpu().numpy()
        _check_step(th0, g_host, m0, v0, t, hp, th1, m.cpu().numpy(), v.cpu().numpy())
        np.testing.assert_array_equal(bf.float().cpu().numpy(), round_to_bf16(th1))
        assert not grad.any()
    assert int(flag.item()) == 0


def test_keeps_gradient_and_skips_bf16_copy_when_asked():
    rng = np.random.default_rng(11)
    n = 4099
    g_host = _grads(rng, n)
    theta, grad = _dev(np.ones(n, np.float32)), _dev(g_host)
    m, v = torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    L.soup_adamw_step(theta, None, grad, m, v, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0, 1, zero_grad=False)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(grad.cpu().numpy(), g_host)


def test_nonfinite_gradient_sets_the_flag():
    rng = np.random.default_rng(12)
    n = 2051
    g_host = _grads(rng, n)
    g_host[1000] = np.inf
    g_host[2050] = np.nan  # in the scalar tail
    theta = _dev((rng.standard_normal(n) * 0.02).astype(np.float32))
    th0 = theta.cpu().numpy()
    m, v, grad = torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda"), _dev(g_host)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, grad_scale=1.0)
    L.soup_adamw_step(theta, None, grad, m, v, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0, 1, nonfinite=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == 1
    ok = np.isfinite(g_host)
    _check_step(th0, g_host, np.zeros(n, np.float32), np.zeros(n, np.float32), 1, hp, theta.cpu().numpy(),
                m.cpu().numpy(), v.cpu().numpy(), idx=ok)


def test_refuses_bad_arguments_without_launching():
    n = 64
    buf = torch.zeros(4 * n + 4, device="cuda")
    th, g, m, v = buf[:n], buf[n:2 * n], buf[2 * n:3 * n], buf[3 * n + 1:4 * n + 1]  # v misaligned
    with pytest.raises(L.SoupError):
        L.soup_adamw_step(th, None, g, m, v, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0, 1)
    with pytest.raises(L.SoupError):
        L.soup_adamw_step(th, None, g, m, buf[3 * n:4 * n], 1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0, 0)  # t = 0
    with pytest.raises(L.SoupError):
        L.soup_adamw_step(th, None, g, m, buf[3 * n:4 * n], 1e-3, 1.0, 0.999, 1e-8, 0.0, 1.0, 1)  # beta1 = 1
    e = torch.empty(0, device="cuda")
    L.soup_adamw_step(e, None, e, e, e, 1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0, 1)  # n = 0: no-op


def test_full_adapter_set_sampled():
    """The Llama-8B adapter set (32 layers, r = 16 on all seven projections,
    41,943,040 parameters in the flat layout) in one launch, as in the
    training step; checked on 200,000 sampled parameters."""
    from layer_streamed_qlora_b200 import dp
    H, I, r, qkv = 4096, 14336, 16, 6144
    shapes = [(3 * r, H), (qkv, r), (r, H), (H, r), (2 * r, H), (2 * I, r), (r, I), (H, r)] * 32
    _, n = dp.flat_layout(shapes)
    assert n == 41_943_040
    gen = torch.Generator(device="cuda").manual_seed(5)
    theta = torch.randn(n, device="cuda", generator=gen) * 0.02
    bf = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    m = torch.randn(n, device="cuda", generator=gen).mul_(1e-3)
    v = torch.rand(n, device="cuda", generator=gen).mul_(1e-6)
    grad = torch.randn(n, device="cuda", generator=gen).mul_(1e-2)
    idx = np.sort(np.random.default_rng(6).choice(n, 200_000, replace=False))
    ti = torch.from_numpy(idx).cuda()
    th0, m0, v0, g0 = (x[ti].cpu().numpy() for x in (theta, m, v, grad))
    hp = dict(lr=5e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, grad_scale=1.0)
    L.soup_adamw_step(theta, bf, grad, m, v, 5e-4, 0.9, 0.999, 1e-8, 0.0, 1.0, 7, zero_grad=True)
    torch.cuda.synchronize()
    th1 = theta[ti].cpu().numpy()
    _check_step(th0, g0, m0, v0, 7, hp, th1, m[ti].cpu().numpy(), v[ti].cpu().numpy())
    np.testing.assert_array_equal(bf[ti].float().cpu().numpy(), round_to_bf16(th1))
    assert not grad.any()


def test_model_optimizer_step_updates_the_factors_the_gemms_read():
    """After a streamed SFT step, StreamedLoRAModel.optimizer_step moves every
    factor by AdamW, rewrites the bf16 factors (the views the layers read) and
    clears the gradients."""
    from layer_streamed_qlora_b200 import model as M
    import soup_synth as ss
    from tests.model_fixture import NumpyWeights
    cfg = M.ModelConfig(hidden=512, n_q_heads=4, n_kv_heads=2, head_dim=128, intermediate=1024, rank=16,
                        alpha=32.0, vocab=512, n_layers=2, kind="nf4")
    B, S = 2, 64
    mdl = M.StreamedLoRAModel(cfg, B, S, n_buffers=2, weights=NumpyWeights(cfg, 0), head_chunk=48)
    try:
        mdl.ids.copy_(torch.from_numpy(ss.uniform_ids(1, "ids", (B, S), cfg.vocab).astype(np.int32)))
        bf_before = mdl.lora_flat.float().cpu().numpy()
        np.testing.assert_array_equal(mdl.master_flat.cpu().numpy(), bf_before)
        for t in (1, 2):
            mdl.sft_step()
            torch.cuda.synchronize()
            th0, g0 = mdl.master_flat.cpu().numpy(), mdl.grad_flat.cpu().numpy()
            m0, v0 = mdl.adam_m.cpu().numpy(), mdl.adam_v.cpu().numpy()
            assert np.abs(g0).max() > 0
            mdl.optimizer_step()
            torch.cuda.synchronize()
            o = mdl.adamw
            hp = dict(lr=o.lr, beta1=o.beta1, beta2=o.beta2, eps=o.eps, weight_decay=o.weight_decay, grad_scale=1.0)
            th1 = mdl.master_flat.cpu().numpy()
            _check_step(th0, g0, m0, v0, t, hp, th1, mdl.adam_m.cpu().numpy(), mdl.adam_v.cpu().numpy())
            np.testing.assert_array_equal(mdl.lora_flat.float().cpu().numpy(), round_to_bf16(th1))
            assert not mdl.grad_flat.any()
        # the per-layer factor views alias the flat buffer the kernel rewrote
        a = mdl.lora[1]["B_gu"]
        off = (a.data_ptr() - mdl.lora_flat.data_ptr()) // 2
        np.testing.assert_array_equal(a.float().cpu().numpy().reshape(-1),
                                      round_to_bf16(th1[off:off + a.numel()]))
        assert int(mdl.nonfinite.item()) == 0
        assert np.any(mdl.lora_flat.float().cpu().numpy() != bf_before)
    finally:
        mdl.close()

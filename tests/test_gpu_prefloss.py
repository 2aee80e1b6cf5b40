"""SimPO and ORPO on the GPU against the oracle.

The loss kernels are compared with the oracle's losses evaluated on the
kernel's own sequence sums (the sums themselves against fp64 sums of the same
log-probs): loss within 1e-5 relative, dL/dlogp within the usual relative
Frobenius 5e-3 / max 1e-2 bound (in practice fp32 rounding).  The streamed
SimPO / ORPO steps of a small model follow the deep-stack comparison
protocol of the DPO test: policy sums against the oracle's forward pass, the
loss and dL/dlogp on the GPU's own sums, every layer against the oracle fed
the GPU's own layer input and upstream gradient, and the end-to-end
gradients at the sanity bound."""
import numpy as np
import pytest
import torch

import soup_synth as ss
from oracle import head as OH
from oracle import layer as OL
from oracle import model as OM
from tests.gpu_util import assert_close
from tests.model_fixture import NumpyWeights, shape_of, split_grads

pytestmark = pytest.mark.gpu
L = None
M = None


@pytest.fixture(scope="module", autouse=True)
def _mods():
    global L, M
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from layer_streamed_qlora_b200 import _lib, model
    _lib.lib()
    L, M = _lib, model
    yield
    assert _lib.device_error() == 0


def _oracle_loss(kind, sums, n, hp):
    c, r = sums[0::2], sums[1::2]
    return OH.simpo_loss(c, r, n, n, *hp) if kind == "simpo" else OH.orpo_loss(c, r, n, n, *hp)


def _run_kernel(kind, logp, pairs, S, P_len, hp, loss, sums, coef):
    if kind == "simpo":
        L.soup_simpo_loss(logp, pairs, S, P_len, hp[0], hp[1], loss, sums, coef)
    else:
        L.soup_orpo_loss(logp, pairs, S, P_len, hp[0], loss, sums, coef)


HP = {"simpo": (2.0, 0.7), "orpo": (0.1,)}


@pytest.mark.parametrize("kind", ["simpo", "orpo"])
@pytest.mark.parametrize("pairs,S,P_len", [(2, 48, 24), (3, 17, 0), (1, 9, 1), (4, 33, 32), (64, 512, 256)])
def test_loss_kernel_matches_oracle(kind, pairs, S, P_len):
    rng = np.random.default_rng(pairs * 1000 + S)
    lp_host = (-rng.random((2 * pairs, S - 1)) * 8).astype(np.float32)
    logp = torch.from_numpy(lp_host).cuda()
    loss = torch.zeros(1, device="cuda")
    sums = torch.zeros(2 * pairs, device="cuda")
    coef = torch.full((2 * pairs, S - 1), 7.0, device="cuda")
    hp = tuple(float(np.float32(h)) for h in HP[kind])
    _run_kernel(kind, logp, pairs, S, P_len, hp, loss, sums, coef)
    torch.cuda.synchronize()
    mask = OM.continuation_mask(S, P_len)
    n = float(mask.sum())
    s_ref = (lp_host.astype(np.float64) * mask[None, :]).sum(axis=1)
    s_gpu = sums.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(s_gpu, s_ref, rtol=1e-5)
    Lr, dc, dr = _oracle_loss(kind, s_gpu, n, hp)
    assert abs(float(loss.item()) - Lr) <= 1e-5 * abs(Lr), (float(loss.item()), Lr)
    d = np.empty(2 * pairs)
    d[0::2], d[1::2] = dc, dr
    c = coef.cpu().numpy()
    assert_close(c, d[:, None] * mask[None, :], f"{kind} dL/dlogp")
    assert not c[:, ~mask].any()  # prompt positions exactly zero


def test_refusals():
    x = torch.zeros((4, 7), device="cuda")
    one = torch.zeros(1, device="cuda")
    for bad in ((0, 8, 2), (2, 1, 0), (2, 8, 8), (2, 8, -1), (4096, 8, 2)):
        with pytest.raises(L.SoupError):
            L.soup_simpo_loss(x, bad[0], bad[1], bad[2], 2.0, 1.0, one, None, x)
        with pytest.raises(L.SoupError):
            L.soup_orpo_loss(x, bad[0], bad[1], bad[2], 0.1, one, None, x)


def _small_cfg():
    return M.ModelConfig(hidden=512, n_q_heads=4, n_kv_heads=2, head_dim=128, intermediate=1024, rank=16,
                         alpha=32.0, vocab=512, n_layers=3, kind="nf4")


@pytest.mark.parametrize("kind", ["simpo", "orpo"])
def test_preference_step_matches_oracle(kind):
    cfg = _small_cfg()
    pairs, P_len, C_len = 2, 24, 24
    S = P_len + C_len
    w = NumpyWeights(cfg, 6)
    m = M.StreamedLoRAModel(cfg, 2 * pairs, S, n_buffers=2, weights=w, head_chunk=48)
    try:
        rows = []
        for p in range(pairs):
            prompt = ss.uniform_ids(20 + p, "prompt", (P_len,), cfg.vocab)
            for which in ("chosen", "rejected"):
                rows.append(np.concatenate([prompt, ss.uniform_ids(20 + p, which, (C_len,), cfg.vocab)]))
        ids = np.stack(rows)
        m.ids.copy_(torch.from_numpy(ids.astype(np.int32)))
        m.capture_dh = {}
        hp = HP[kind]
        loss = float((m.simpo_step(P_len, *hp) if kind == "simpo" else m.orpo_step(P_len, *hp)).item())
        torch.cuda.synchronize()
        P = w.oracle_params()
        shape = shape_of(cfg)
        step = OM.simpo_step if kind == "simpo" else OM.orpo_step
        lo, grads, ex = step(P, ids, shape, P_len, *hp)
        sums = m.seq_sums.cpu().numpy().astype(np.float64)[:2 * pairs]
        assert_close(sums, ex["policy"], f"{kind} policy seq logp")
        mask = OM.continuation_mask(S, P_len)
        n = float(mask.sum())
        hp32 = tuple(float(np.float32(h)) for h in hp)
        L_own, dc, dr = _oracle_loss(kind, sums, n, hp32)
        assert abs(loss - L_own) <= 1e-5 * abs(L_own), (loss, L_own)
        coef = np.zeros((2 * pairs, S - 1))
        coef[0::2] = dc[:, None] * mask[None, :]
        coef[1::2] = dr[:, None] * mask[None, :]
        assert_close(m.coef.cpu().numpy(), coef, f"{kind} dL/dlogp")
        # every layer against the oracle fed the GPU's own layer input and upstream gradient
        B, H = 2 * pairs, cfg.hidden
        for l in range(cfg.n_layers):
            Wd, lora = P["layers"][l]
            h_in = m.ckpt[l].float().cpu().numpy().astype(np.float64).reshape(B, S, H)
            out, cache = OL.layer_fwd(h_in, Wd, lora, shape)
            assert_close(m.ckpt[l + 1].float().cpu().numpy().reshape(B, S, H), out, f"L{l} h_out")
            dh_out = m.capture_dh[l + 1].cpu().numpy().astype(np.float64).reshape(B, S, H)
            dh_in, g_l = OL.layer_bwd(cache, Wd, lora, shape, dh_out)
            assert_close(m.capture_dh[l].cpu().numpy().reshape(B, S, H), dh_in, f"L{l} dh_in")
            got = split_grads(cfg, m.grads[l])
            for p in ss.PROJ_NAMES:
                assert_close(got[p][0], g_l[p][0], f"L{l} dA_{p}")
                assert_close(got[p][1], g_l[p][1], f"L{l} dB_{p}")
        # end to end (compounded over the stack): sanity bound
        assert abs(loss - lo) <= 2e-2 * abs(lo), (loss, lo)
        for l in range(cfg.n_layers):
            got = split_grads(cfg, m.grads[l])
            for p in ss.PROJ_NAMES:
                assert_close(got[p][0], grads[l][p][0], f"e2e L{l} dA_{p}", rel=2e-2, maxrel=5e-2)
                assert_close(got[p][1], grads[l][p][1], f"e2e L{l} dB_{p}", rel=2e-2, maxrel=5e-2)
    finally:
        m.close()

"""The whole streamed step on the GPU (embedding gather, streamed decoder
layers, chunked head, CE / DPO, recompute backward) against the CPU oracle at
reduced depth and width, plus the pages' bit-exactness protocol: streamed runs
(stream_buffers 2, 4, 8 and an all-resident ring) give the same bits.

Deep stacks compound bf16 rounding layer after layer, so (reading of the
comparison protocol) every layer is checked against the
oracle fed the GPU's own bf16 layer input and fp32 upstream gradient, the head
against the oracle on the GPU's final hidden state, and the DPO loss against
the DPO formula on the GPU's own sequence sums, each within relative Frobenius
5e-3 and max|diff| 1e-2 max|ref|; the end-to-end CE loss is held to 5e-3 and
the end-to-end gradients and DPO loss to a sanity bound of 2e-2."""
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
M = None


@pytest.fixture(scope="module", autouse=True)
def _mods():
    global M
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from layer_streamed_qlora_b200 import _lib, model
    _lib.lib()
    M = model
    yield
    assert _lib.device_error() == 0


def small_cfg(kind="nf4", tied=False, n_layers=3):
    # reduced Llama-style shape: 4 q / 2 kv heads of 128 (GQA group 2), SwiGLU 1024
    return M.ModelConfig(hidden=512, n_q_heads=4, n_kv_heads=2, head_dim=128, intermediate=1024, rank=16,
                         alpha=32.0, vocab=512, n_layers=n_layers, kind=kind, tied=tied)


def build(cfg, B, S, n_buffers=2, seed=0, chunk=48, task="sft", recompute="auto", prompt_dedup=0):
    w = NumpyWeights(cfg, seed)
    m = M.StreamedLoRAModel(cfg, B, S, n_buffers=n_buffers, weights=w, head_chunk=chunk, task=task,
                            stream_recompute=recompute, prompt_dedup=prompt_dedup)
    return m, w


def set_ids(m, ids):
    m.set_ids(torch.from_numpy(ids.astype(np.int32)))  # the model also lays out the shared-prompt rows
    torch.cuda.synchronize()


def check_layers_on_gpu_inputs(m, w, cfg):
    """Layer-by-layer: oracle fed the GPU's own layer input and upstream grad."""
    shape = shape_of(cfg)
    P = w.oracle_params()
    B, S, H = m.batch, m.seq, cfg.hidden
    for l in range(cfg.n_layers):
        Wd, lora = P["layers"][l]
        h_in = m.ckpt[l].float().cpu().numpy().astype(np.float64).reshape(B, S, H)
        out, cache = OL.layer_fwd(h_in, Wd, lora, shape)
        assert_close(m.ckpt[l + 1].float().cpu().numpy().reshape(B, S, H), out, f"L{l} h_out")
        dh_out = m.capture_dh[l + 1].cpu().numpy().astype(np.float64).reshape(B, S, H)
        dh_in, grads = OL.layer_bwd(cache, Wd, lora, shape, dh_out)
        assert_close(m.capture_dh[l].cpu().numpy().reshape(B, S, H), dh_in, f"L{l} dh_in")
        got = split_grads(cfg, m.grads[l])
        for p in ss.PROJ_NAMES:
            assert_close(got[p][0], grads[p][0], f"L{l} dA_{p}")
            assert_close(got[p][1], grads[p][1], f"L{l} dB_{p}")


@pytest.mark.parametrize("kind,tied,recompute", [("nf4", False, "auto"), ("bf16", True, "auto"),
                                                ("nf4", False, "recompute")])
def test_sft_step_matches_oracle(kind, tied, recompute):
    """recompute="auto" (uncapped): every layer keeps its activations (no
    forward recompute in the backward); "recompute": none kept."""
    cfg = small_cfg(kind, tied)
    B, S = 2, 64
    m, w = build(cfg, B, S, recompute=recompute)
    assert m.keep_plan == (["saved"] * cfg.n_layers if recompute == "auto" else [None] * cfg.n_layers)
    m.capture_dh = {}
    ids = ss.uniform_ids(1, "ids", (B, S), cfg.vocab)
    set_ids(m, ids)
    loss = float(m.sft_step().item())
    P = w.oracle_params()
    lo, grads, _ = OM.sft_step(P, ids, shape_of(cfg))
    assert abs(loss - lo) <= 5e-3 * abs(lo), (loss, lo)
    # head on the GPU's own final hidden state
    hL = m.ckpt[cfg.n_layers].float().cpu().numpy().astype(np.float64).reshape(B, S, cfg.hidden)
    logp, hc = OH.token_logprobs(hL, P["final_norm"], P["head"], ids, cfg.eps)
    assert_close(m.logp.cpu().numpy(), logp, "logp")
    _, dlogp = OH.ce_loss(logp)
    dh_top = OH.token_logprobs_bwd(hc, P["final_norm"], P["head"], ids, dlogp)
    assert_close(m.capture_dh[cfg.n_layers].cpu().numpy().reshape(dh_top.shape), dh_top, "dh(head)")
    check_layers_on_gpu_inputs(m, w, cfg)
    # end to end (compounded over the stack): sanity bound
    for l in range(cfg.n_layers):
        got = split_grads(cfg, m.grads[l])
        for p in ss.PROJ_NAMES:
            assert_close(got[p][0], grads[l][p][0], f"e2e L{l} dA_{p}", rel=2e-2, maxrel=5e-2)
            assert_close(got[p][1], grads[l][p][1], f"e2e L{l} dB_{p}", rel=2e-2, maxrel=5e-2)
    m.close()


def test_streamed_equals_resident_bit_exact():
    cfg = small_cfg("nf4", False, n_layers=4)
    B, S = 2, 64
    ids = ss.uniform_ids(2, "ids", (B, S), cfg.vocab)
    ref = None
    for nb in (2, 4, 8):  # 8 >= n_layers: every layer stays resident after its first read
        m, _ = build(cfg, B, S, n_buffers=nb, seed=3)
        set_ids(m, ids)
        out = []
        for _ in range(2):  # second step exercises reuse across steps
            loss = m.sft_step().clone()
            torch.cuda.synchronize()
            out.append((loss.cpu(), [{k: v.cpu().clone() for k, v in g.items()} for g in m.grads],
                        m.logp.cpu().clone()))
        st = m.plan.stats()
        if nb >= cfg.n_layers:
            assert st["copies"] <= cfg.n_layers + 2  # layers read once, plus the lm_head
        m.close()
        if ref is None:
            ref = out
            continue
        for (l1, g1, p1), (l2, g2, p2) in zip(ref, out):
            assert torch.equal(l1, l2), (nb, l1, l2)
            assert torch.equal(p1, p2), nb
            for a, b in zip(g1, g2):
                for k in a:
                    assert torch.equal(a[k], b[k]), (nb, k)


def test_dpo_step_matches_oracle():
    cfg = small_cfg("nf4", False)
    pairs, P_len, C_len = 2, 24, 24
    S = P_len + C_len
    m, w = build(cfg, 2 * pairs, S, seed=5)
    g = np.random.default_rng(7)
    rows = []
    for p in range(pairs):
        prompt = ss.uniform_ids(10 + p, "prompt", (P_len,), cfg.vocab)
        for which in ("chosen", "rejected"):
            cont = ss.uniform_ids(10 + p, which, (C_len,), cfg.vocab)
            rows.append(np.concatenate([prompt, cont]))
    ids = np.stack(rows)
    set_ids(m, ids)
    m.capture_dh = {}
    loss = float(m.dpo_step(P_len, 0.1).item())
    P = w.oracle_params()
    lo, grads, ex = OM.dpo_step(P, ids, shape_of(cfg), P_len, 0.1)
    sums = m.seq_sums.cpu().numpy().astype(np.float64)
    assert_close(sums[:2 * pairs], ex["policy"], "policy seq logp")
    assert_close(sums[2 * pairs:], ex["reference"], "reference seq logp")
    # the DPO loss and its coefficients on the GPU's own sequence sums
    pol, ref = sums[:2 * pairs], sums[2 * pairs:]
    L_own, dc, dr = OH.dpo_loss(pol[0::2], pol[1::2], ref[0::2], ref[1::2], 0.1)
    assert abs(loss - L_own) <= 1e-5 * abs(L_own), (loss, L_own)
    mask = OM.continuation_mask(S, P_len)
    coef = np.zeros((2 * pairs, S - 1))
    coef[0::2] = dc[:, None] * mask[None, :]
    coef[1::2] = dr[:, None] * mask[None, :]
    assert_close(m.coef.cpu().numpy(), coef, "DPO dL/dlogp")
    check_layers_on_gpu_inputs(m, w, cfg)
    # end to end: a difference of nearly equal sums amplifies their rounding
    assert abs(loss - lo) <= 2e-2 * abs(lo), (loss, lo)
    for l in range(cfg.n_layers):
        got = split_grads(cfg, m.grads[l])
        for p in ss.PROJ_NAMES:
            assert_close(got[p][0], grads[l][p][0], f"e2e L{l} dA_{p}", rel=2e-2, maxrel=5e-2)
            assert_close(got[p][1], grads[l][p][1], f"e2e L{l} dB_{p}", rel=2e-2, maxrel=5e-2)
    m.close()


def _dpo_ids(cfg, pairs, P_len, C_len, seed=10):
    rows = []
    for p in range(pairs):
        prompt = ss.uniform_ids(seed + p, "prompt", (P_len,), cfg.vocab)
        for which in ("chosen", "rejected"):
            rows.append(np.concatenate([prompt, ss.uniform_ids(seed + p, which, (C_len,), cfg.vocab)]))
    return np.stack(rows)


def test_dpo_shared_visit_equals_two_passes_bit_exact():
    """task="dpo" runs the reference and the policy forward pass in one visit
    per layer: the same bits as the two separate streamed passes, with fewer
    layer copies."""
    cfg = small_cfg("nf4", False, n_layers=4)
    pairs, P_len, C_len = 2, 24, 24
    ids = _dpo_ids(cfg, pairs, P_len, C_len)
    out = {}
    for task in ("sft", "dpo"):  # "sft": a model without the shared-visit buffers
        m, _ = build(cfg, 2 * pairs, P_len + C_len, seed=5, task=task)
        set_ids(m, ids)
        m.plan.reset_stats()
        loss = m.dpo_step(P_len, 0.1).clone()
        torch.cuda.synchronize()
        out[task] = (loss, m.logp.clone(), m.logp_ref.clone(), m.seq_sums.clone(), m.grad_flat.clone(),
                     m.plan.stats()["copies"])
        m.close()
    a, b = out["sft"], out["dpo"]
    for x, y, name in zip(a[:5], b[:5], ("loss", "logp", "logp_ref", "seq_sums", "grads")):
        assert torch.equal(x, y), name
    assert b[5] < a[5], (a[5], b[5])


@pytest.mark.parametrize("task", ["dpo", "simpo"])
def test_prompt_dedup_matches_the_plain_preference_step(task):
    """Pairs whose 128-token prompt is stored and computed once per pair (the
    pair's token rows are [prompt | chosen | rejected continuation]) give the
    preference step of the plain layout: the loss, the four sequence sums and
    every LoRA gradient within the tolerances (different reduction orders, the
    same quantities), with 32 % fewer token rows; and the loss and gradients
    match the oracle's step end to end."""
    cfg = small_cfg("nf4", False, n_layers=3)
    pairs, P_len, C_len = 2, 128, 72
    S = P_len + C_len
    ids = _dpo_ids(cfg, pairs, P_len, C_len)
    out = {}
    for dd in (0, P_len):
        m, w = build(cfg, 2 * pairs, S, seed=5, task=task, prompt_dedup=dd)
        set_ids(m, ids)
        loss = m.dpo_step(P_len, 0.1) if task == "dpo" else m.simpo_step(P_len, 2.0, 1.0)
        torch.cuda.synchronize()
        out[dd] = (float(loss.item()), m.seq_sums.cpu().numpy().astype(np.float64)[:4 * pairs],
                   [split_grads(cfg, g) for g in m.grads], m.T)
        m.close()
    (l0, s0, g0, t0), (l1, s1, g1, t1) = out[0], out[P_len]
    assert t0 == 2 * pairs * S and t1 == pairs * (P_len + 2 * C_len)
    assert abs(l1 - l0) <= 1e-3 * max(1.0, abs(l0)), (l0, l1)
    n = 4 * pairs if task == "dpo" else 2 * pairs
    assert_close(s1[:n], s0[:n], "sequence sums")
    for l in range(cfg.n_layers):
        for p in ss.PROJ_NAMES:
            assert_close(g1[l][p][0], g0[l][p][0], f"L{l} dA_{p}")
            assert_close(g1[l][p][1], g0[l][p][1], f"L{l} dB_{p}")
    if task == "dpo":
        P = w.oracle_params()
        lo, grads, _ = OM.dpo_step(P, ids, shape_of(cfg), P_len, 0.1)
        assert abs(l1 - lo) <= 2e-2 * abs(lo), (l1, lo)
        for l in range(cfg.n_layers):
            for p in ss.PROJ_NAMES:
                assert_close(g1[l][p][0], grads[l][p][0], f"e2e L{l} dA_{p}", rel=2e-2, maxrel=5e-2)
                assert_close(g1[l][p][1], grads[l][p][1], f"e2e L{l} dB_{p}", rel=2e-2, maxrel=5e-2)


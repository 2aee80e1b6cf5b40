"""Pins for the head / loss / DPO / whole-stack oracle (CPU): closed forms
(uniform logits give log V; policy == reference gives log 2), finite
differences through the head and through a tiny stack for both SFT and DPO,
and chunking invariance of the loss."""
import numpy as np

import soup_synth as ss
from oracle import head as Hd
from oracle import model as M


def test_uniform_logits_give_log_vocab():
    V, H = 11, 8
    ids = np.random.default_rng(0).integers(0, V, (2, 6))
    h = np.random.default_rng(1).standard_normal((2, 6, H))
    logp, _ = Hd.token_logprobs(h, np.ones(H), np.zeros((V, H)), ids, 1e-5)
    loss, _ = Hd.ce_loss(logp)
    np.testing.assert_allclose(loss, np.log(V), rtol=1e-14)


def test_head_finite_differences_and_chunking():
    V, H = 13, 8
    g = np.random.default_rng(2)
    ids = g.integers(0, V, (2, 7))
    h = g.standard_normal((2, 7, H)); E = g.standard_normal((V, H)); w = 1 + 0.1 * g.standard_normal(H)
    dl = g.standard_normal((2, 6))
    f = lambda h_: float(np.sum(Hd.token_logprobs(h_, w, E, ids, 1e-5)[0] * dl))
    lp, cache = Hd.token_logprobs(h, w, E, ids, 1e-5)
    lp2, _ = Hd.token_logprobs(h, w, E, ids, 1e-5, chunk=2)
    np.testing.assert_allclose(lp, lp2, rtol=1e-13, atol=1e-13)
    dh = Hd.token_logprobs_bwd(cache, w, E, ids, dl)
    eps = 1e-6
    for _ in range(4):
        v = g.standard_normal(h.shape)
        num = (f(h + eps * v) - f(h - eps * v)) / (2 * eps)
        assert abs(num - np.sum(dh * v)) < 1e-6 * max(1, abs(num))


def test_dpo_at_reference_is_log2():
    pol = np.array([-3.0, -7.0, -1.5, -2.0])
    loss, dc, dr = Hd.dpo_loss(pol[0::2], pol[1::2], pol[0::2], pol[1::2], 0.1)
    np.testing.assert_allclose(loss, np.log(2.0), rtol=1e-15)
    np.testing.assert_allclose(dc, -0.1 * 0.5 / 2, rtol=1e-15)
    np.testing.assert_allclose(dr, 0.1 * 0.5 / 2, rtol=1e-15)


def test_dpo_finite_differences():
    g = np.random.default_rng(3)
    pc, pr, rc, rr = (g.standard_normal(4) * 5 for _ in range(4))
    loss, dc, dr = Hd.dpo_loss(pc, pr, rc, rr, 0.1)
    eps = 1e-6
    for i in range(4):
        e = np.zeros(4); e[i] = eps
        nc = (Hd.dpo_loss(pc + e, pr, rc, rr, 0.1)[0] - Hd.dpo_loss(pc - e, pr, rc, rr, 0.1)[0]) / (2 * eps)
        nr = (Hd.dpo_loss(pc, pr + e, rc, rr, 0.1)[0] - Hd.dpo_loss(pc, pr - e, rc, rr, 0.1)[0]) / (2 * eps)
        assert abs(nc - dc[i]) < 1e-8 and abs(nr - dr[i]) < 1e-8


def _tiny_params(shape, seed, tied=False):
    g = np.random.default_rng(seed)
    layers = []
    for _ in range(shape.n_layers):
        W = {p: g.standard_normal(shape.proj_shape(p)) * 0.2 for p in ss.PROJ_NAMES}
        W["norm1"] = 1 + 0.1 * g.standard_normal(shape.hidden)
        W["norm2"] = 1 + 0.1 * g.standard_normal(shape.hidden)
        lora = {}
        for p in ss.PROJ_NAMES:
            o, i = shape.proj_shape(p)
            lora[p] = (g.standard_normal((shape.rank, i)) * 0.3, g.standard_normal((o, shape.rank)) * 0.3)
        layers.append((W, lora))
    E = g.standard_normal((shape.vocab, shape.hidden))
    head = E if tied else g.standard_normal((shape.vocab, shape.hidden))
    return dict(layers=layers, embed=E, head=head, final_norm=1 + 0.1 * g.standard_normal(shape.hidden))


SHAPE = ss.tiny_layer_shape(hidden=16, n_q=4, n_kv=2, head_dim=4, inter=24, rank=2, alpha=4.0,
                            vocab=19, n_layers=2)


def _perturbed(params, li, p, which, delta):
    layers = []
    for j, (W, lora) in enumerate(params["layers"]):
        if j == li:
            lora = dict(lora)
            pair = list(lora[p]); pair[which] = pair[which] + delta; lora[p] = tuple(pair)
        layers.append((W, lora))
    out = dict(params); out["layers"] = layers
    return out


def test_sft_stack_finite_differences():
    params = _tiny_params(SHAPE, 4)
    ids = np.random.default_rng(5).integers(0, SHAPE.vocab, (2, 6))
    loss, grads, _ = M.sft_step(params, ids, SHAPE)
    g = np.random.default_rng(6)
    eps = 1e-6
    for li, p, which in ((0, "q", 0), (1, "down", 1), (0, "up", 1), (1, "v", 0)):
        v = g.standard_normal(params["layers"][li][1][p][which].shape)
        lp = M.sft_step(_perturbed(params, li, p, which, eps * v), ids, SHAPE)[0]
        lm = M.sft_step(_perturbed(params, li, p, which, -eps * v), ids, SHAPE)[0]
        num = (lp - lm) / (2 * eps)
        ana = float(np.sum(grads[li][p][which] * v))
        assert abs(num - ana) < 1e-6 * max(1, abs(ana)), (li, p, which, num, ana)


def test_dpo_stack_finite_differences_and_reference():
    params = _tiny_params(SHAPE, 7, tied=True)
    g = np.random.default_rng(8)
    prompt = g.integers(0, SHAPE.vocab, 3)
    ids = np.stack([np.concatenate([prompt, g.integers(0, SHAPE.vocab, 3)]) for _ in range(4)])
    ids[2:, :3] = g.integers(0, SHAPE.vocab, 3)     # a second pair with its own prompt
    loss, grads, ex = M.dpo_step(params, ids, SHAPE, prompt_len=3, beta=0.1)
    # the reference pass is the same stack with adapters off == every B zeroed
    zeroB = dict(params)
    zeroB["layers"] = [(W, {p: (A, np.zeros_like(B)) for p, (A, B) in lora.items()})
                       for W, lora in params["layers"]]
    ref2, _ = M.seq_logprob_sums(zeroB, ids, SHAPE, 3, adapters_on=True)
    assert np.array_equal(ex["reference"], ref2)
    eps = 1e-6
    for li, p, which in ((0, "k", 1), (1, "gate", 0)):
        v = g.standard_normal(params["layers"][li][1][p][which].shape)
        lp = M.dpo_step(_perturbed(params, li, p, which, eps * v), ids, SHAPE, 3, 0.1)[0]
        lm = M.dpo_step(_perturbed(params, li, p, which, -eps * v), ids, SHAPE, 3, 0.1)[0]
        num = (lp - lm) / (2 * eps)
        ana = float(np.sum(grads[li][p][which] * v))
        assert abs(num - ana) < 1e-6 * max(1e-3, abs(ana)), (li, p, which, num, ana)

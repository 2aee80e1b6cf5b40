"""Pins for the head / loss / DPO / SimPO / ORPO / whole-stack oracle (CPU):
closed forms (uniform logits give log V; policy == reference gives log 2;
SimPO with one-token continuations is DPO with a zero reference; ORPO at
odds 1 vs 1/3 by hand), finite differences through the losses, the head and
a tiny stack for SFT, DPO, SimPO and ORPO, and chunking invariance of the
loss."""
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


def _fd_pairs(fn, pc, pr, eps=1e-6):
    loss, dc, dr = fn(pc, pr)
    for i in range(pc.size):
        e = np.zeros(pc.size); e[i] = eps
        nc = (fn(pc + e, pr)[0] - fn(pc - e, pr)[0]) / (2 * eps)
        nr = (fn(pc, pr + e)[0] - fn(pc, pr - e)[0]) / (2 * eps)
        assert abs(nc - dc[i]) < 1e-8 and abs(nr - dr[i]) < 1e-8, (i, nc, dc[i], nr, dr[i])


def test_simpo_closed_forms_and_finite_differences():
    n = 7.0
    pc = np.array([-21.0, -3.5, -40.0])
    # equal normalised log-likelihoods and gamma = 0: log 2, gradients -/+ beta / (2 P n)
    loss, dc, dr = Hd.simpo_loss(pc, pc, n, n, 2.0, 0.0)
    np.testing.assert_allclose(loss, np.log(2.0), rtol=1e-15)
    np.testing.assert_allclose(dc, -2.0 * 0.5 / (3 * n), rtol=1e-15)
    np.testing.assert_allclose(dr, 2.0 * 0.5 / (3 * n), rtol=1e-15)
    # one-token continuations, gamma = 0: the DPO loss with a zero reference
    pr = np.array([-20.0, -4.0, -41.5])
    ls, sc, sr = Hd.simpo_loss(pc, pr, 1.0, 1.0, 0.3, 0.0)
    ld, qc, qr = Hd.dpo_loss(pc, pr, np.zeros(3), np.zeros(3), 0.3)
    np.testing.assert_allclose([ls, *sc, *sr], [ld, *qc, *qr], rtol=1e-14)
    # the target margin: z = beta (m_c - m_r) - gamma exactly 0 gives log 2
    np.testing.assert_allclose(Hd.simpo_loss(np.array([-7.0]), np.array([-14.0]), 7.0, 7.0, 2.0, 2.0)[0],
                               np.log(2.0), rtol=1e-15)
    g = np.random.default_rng(9)
    _fd_pairs(lambda a, b: Hd.simpo_loss(a, b, 5.0, 5.0, 2.0, 1.0), g.standard_normal(4) * 8 - 20,
              g.standard_normal(4) * 8 - 20)


def test_orpo_closed_forms_and_finite_differences():
    # P = 1, mean log-likelihoods log(1/2) (odds 1) and log(1/4) (odds 1/3):
    # log odds ratio = log 3, so L = -log(1/2) + lam * -log(3/4)
    n, lam = 4.0, 0.1
    pc, pr = np.array([n * np.log(0.5)]), np.array([n * np.log(0.25)])
    loss, dc, dr = Hd.orpo_loss(pc, pr, n, n, lam)
    np.testing.assert_allclose(loss, np.log(2.0) + lam * np.log(4.0 / 3.0), rtol=1e-14)
    # sigmoid(-log 3) = 1/4; d log odds / dm = 1/(1 - e^m): 2 (chosen), 4/3 (rejected)
    np.testing.assert_allclose(dc, (-1.0 - lam * 0.25 * 2.0) / n, rtol=1e-14)
    np.testing.assert_allclose(dr, (lam * 0.25 * 4.0 / 3.0) / n, rtol=1e-14)
    # lam = 0: the chosen continuation's mean NLL only
    pcs, prs = np.array([-30.0, -12.0]), np.array([-25.0, -50.0])
    loss0, dc0, dr0 = Hd.orpo_loss(pcs, prs, 10.0, 10.0, 0.0)
    np.testing.assert_allclose(loss0, (3.0 + 1.2) / 2, rtol=1e-15)
    np.testing.assert_allclose(dc0, -1.0 / 20.0, rtol=1e-15)
    assert not dr0.any()
    # identical sequences: the odds-ratio term is lam log 2
    np.testing.assert_allclose(Hd.orpo_loss(pcs, pcs, 10.0, 10.0, lam)[0], 2.1 + lam * np.log(2.0), rtol=1e-14)
    # both branches of log(1 - e^m): m just below 0 and far below
    g = np.random.default_rng(10)
    _fd_pairs(lambda a, b: Hd.orpo_loss(a, b, 6.0, 6.0, 0.5), np.array([-0.05, -3.0, -60.0, -4.1]),
              np.array([-2.0, -0.3, -55.0, -90.0]))
    _fd_pairs(lambda a, b: Hd.orpo_loss(a, b, 3.0, 3.0, 0.1), g.standard_normal(3) * 3 - 9,
              g.standard_normal(3) * 3 - 9)


def _pref_ids(g):
    prompt = g.integers(0, SHAPE.vocab, 3)
    ids = np.stack([np.concatenate([prompt, g.integers(0, SHAPE.vocab, 3)]) for _ in range(4)])
    ids[2:, :3] = g.integers(0, SHAPE.vocab, 3)
    return ids


def test_simpo_and_orpo_stack_finite_differences():
    params = _tiny_params(SHAPE, 11)
    ids = _pref_ids(np.random.default_rng(12))
    g = np.random.default_rng(13)
    eps = 1e-6
    for step in (lambda P_: M.simpo_step(P_, ids, SHAPE, 3, 2.0, 0.5),
                 lambda P_: M.orpo_step(P_, ids, SHAPE, 3, 0.1)):
        loss, grads, ex = step(params)
        assert ex["policy"].shape == (4,)
        for li, p, which in ((0, "o", 1), (1, "q", 0)):
            v = g.standard_normal(params["layers"][li][1][p][which].shape)
            lp = step(_perturbed(params, li, p, which, eps * v))[0]
            lm = step(_perturbed(params, li, p, which, -eps * v))[0]
            num = (lp - lm) / (2 * eps)
            ana = float(np.sum(grads[li][p][which] * v))
            assert abs(num - ana) < 1e-6 * max(1e-3, abs(ana)), (li, p, which, num, ana)

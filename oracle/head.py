"""Embedding, output head, next-token cross-entropy and DPO
(oracle; test infrastructure only).

* The vocab-sized ``embed_tokens`` and (untied) ``lm_head`` are the two
  tensors that share the vocab slot on the Soup pages ("how layer streaming
  works"); with tied embeddings they are the same matrix.
* SFT loss: mean next-token cross-entropy over the B*(S-1) predicted positions
  of each batch (the pages' ``stream_loss_chunk`` computes the same loss a
  chunk of tokens at a time; chunking does not change the value).
* DPO (the preference loss the pages stream with an adapters-off reference,
  "memory-free reference model"): the plain loss of Rafailov et al. (2023),
    L = -(1/P) sum_p log sigmoid(beta [(pi_c - ref_c) - (pi_r - ref_r)]),
  where pi_* / ref_* are the summed next-token log-probabilities of the
  chosen / rejected continuation tokens under the policy (adapters on) and the
  reference (adapters off).  Prompt positions are masked out.
* SimPO and ORPO, the reference-free preference losses the pages name as the
  ones without DPO's extra reference reads ("memory-free reference model"):
  SimPO (Meng, Xia & Chen 2024) and ORPO (Hong, Lee & Thorne 2024), both on
  length-normalised continuation log-likelihoods (see their functions).
fp64 throughout.
"""
from __future__ import annotations

import numpy as np

from .layer import rmsnorm_bwd, rmsnorm_fwd


def embed(ids, E):
    return np.asarray(E, np.float64)[np.asarray(ids)]


def embed_bwd_rows(ids, dh, vocab):
    """Gradient w.r.t. the embedding matrix (unused by LoRA training, which
    freezes it; kept for tests of the gather)."""
    dE = np.zeros((vocab, dh.shape[-1]))
    np.add.at(dE, np.asarray(ids).reshape(-1), dh.reshape(-1, dh.shape[-1]))
    return dE


def _logsumexp(z):
    m = z.max(axis=-1, keepdims=True)
    return (m + np.log(np.exp(z - m).sum(axis=-1, keepdims=True)))[..., 0]


def token_logprobs(h, w_final, E_head, ids, eps, chunk=256):
    """log p(ids[b, t+1] | prefix) for t = 0..S-2, shape [B, S-1].
    Returns (logp, cache)."""
    h = np.asarray(h, np.float64)
    Bsz, S, H = h.shape
    x, rinv = rmsnorm_fwd(h, w_final, eps)
    E = np.asarray(E_head, np.float64)
    logp = np.empty((Bsz, S - 1))
    for b in range(Bsz):
        for t0 in range(0, S - 1, chunk):
            t1 = min(S - 1, t0 + chunk)
            z = x[b, t0:t1] @ E.T
            lab = np.asarray(ids)[b, t0 + 1:t1 + 1]
            logp[b, t0:t1] = z[np.arange(t1 - t0), lab] - _logsumexp(z)
    return logp, dict(h=h, x=x, rinv=rinv)


def token_logprobs_bwd(cache, w_final, E_head, ids, dlogp, chunk=256):
    """dL/dh given dL/dlogp [B, S-1]."""
    h, x, rinv = cache["h"], cache["x"], cache["rinv"]
    Bsz, S, H = h.shape
    E = np.asarray(E_head, np.float64)
    dx = np.zeros_like(x)
    for b in range(Bsz):
        for t0 in range(0, S - 1, chunk):
            t1 = min(S - 1, t0 + chunk)
            z = x[b, t0:t1] @ E.T
            p = np.exp(z - _logsumexp(z)[:, None])
            lab = np.asarray(ids)[b, t0 + 1:t1 + 1]
            c = np.asarray(dlogp, np.float64)[b, t0:t1]
            dz = -p * c[:, None]
            dz[np.arange(t1 - t0), lab] += c
            dx[b, t0:t1] = dz @ E
    return rmsnorm_bwd(h, w_final, rinv, dx)


def ce_loss(logp):
    """Mean next-token cross-entropy and its gradient w.r.t. logp."""
    n = logp.size
    return -float(np.sum(logp)) / n, np.full(logp.shape, -1.0 / n)


def dpo_loss(pi_c, pi_r, ref_c, ref_r, beta):
    """DPO loss over P pairs and its gradient w.r.t. the policy sums.
    Returns (loss, dL/dpi_c [P], dL/dpi_r [P])."""
    pi_c, pi_r = np.asarray(pi_c, np.float64), np.asarray(pi_r, np.float64)
    z = beta * ((pi_c - np.asarray(ref_c)) - (pi_r - np.asarray(ref_r)))
    P = z.shape[0]
    # -log sigmoid(z) = softplus(-z), computed stably
    loss = float(np.sum(np.logaddexp(0.0, -z))) / P
    dz = -(0.5 * (1.0 - np.tanh(0.5 * z))) / P        # d/dz softplus(-z) = -sigmoid(-z)
    return loss, beta * dz, -beta * dz


def _sigmoid_neg(z):
    """sigmoid(-z), computed without overflow."""
    return 0.5 * (1.0 - np.tanh(0.5 * z))


def _log1mexp(m):
    """log(1 - exp(m)) for m < 0 (Maechler's two-branch form, accurate on both
    sides of m = -log 2)."""
    m = np.asarray(m, np.float64)
    return np.where(m > -np.log(2.0), np.log(-np.expm1(m)), np.log1p(-np.exp(m)))


def simpo_loss(pi_c, pi_r, n_c, n_r, beta, gamma):
    """SimPO over P pairs: with the length-normalised sequence log-likelihoods
    m = pi / n (pi the summed continuation log-probs, n the continuation
    length),
      L = -(1/P) sum_p log sigmoid(beta (m_c - m_r) - gamma).
    Returns (loss, dL/dpi_c [P], dL/dpi_r [P])."""
    pi_c, pi_r = np.asarray(pi_c, np.float64), np.asarray(pi_r, np.float64)
    z = beta * (pi_c / n_c - pi_r / n_r) - gamma
    P = z.shape[0]
    loss = float(np.sum(np.logaddexp(0.0, -z))) / P
    dz = -_sigmoid_neg(z) / P
    return loss, beta * dz / n_c, -beta * dz / n_r


def orpo_loss(pi_c, pi_r, n_c, n_r, lam):
    """ORPO over P pairs: the chosen continuation's mean token NLL plus lam
    times the odds-ratio term.  With m = pi / n the length-normalised
    log-likelihood, odds(y) = exp(m) / (1 - exp(m)), so
    log odds = m - log(1 - exp(m)), and
      L = (1/P) sum_p [ -m_c - lam log sigmoid(log odds_c - log odds_r) ].
    Returns (loss, dL/dpi_c [P], dL/dpi_r [P]); d(log odds)/dm = 1 / (1 - exp(m))."""
    pi_c, pi_r = np.asarray(pi_c, np.float64), np.asarray(pi_r, np.float64)
    m_c, m_r = pi_c / n_c, pi_r / n_r
    z = (m_c - _log1mexp(m_c)) - (m_r - _log1mexp(m_r))
    P = z.shape[0]
    loss = (float(np.sum(-m_c)) + lam * float(np.sum(np.logaddexp(0.0, -z)))) / P
    s = _sigmoid_neg(z)
    dm_c = (-1.0 - lam * s / -np.expm1(m_c)) / P
    dm_r = (lam * s / -np.expm1(m_r)) / P
    return loss, dm_c / n_c, dm_r / n_r

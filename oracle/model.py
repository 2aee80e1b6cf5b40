"""The whole LoRA-adapted stack for one SFT, DPO, SimPO or ORPO step
(oracle; test infrastructure only).

Streaming (one layer in VRAM at a time, each layer read for the forward pass
and again for the recompute; Soup pages, "how layer streaming works") does not
change what is computed, so this is the plain resident computation:
embed -> L decoder layers -> final RMSNorm -> lm_head -> loss, with the hand
written backward of ``oracle.layer`` and ``oracle.head``.  Only the LoRA
factors receive gradients.
"""
from __future__ import annotations

import numpy as np

from .head import ce_loss, dpo_loss, embed, orpo_loss, simpo_loss, token_logprobs, token_logprobs_bwd
from .layer import layer_bwd, layer_fwd


def stack_fwd(params, ids, shape, adapters_on=True, keep=True):
    h = embed(ids, params["embed"])
    caches, inputs = [], []
    for Wl, Ll in params["layers"]:
        inputs.append(h)
        h, c = layer_fwd(h, Wl, Ll, shape, adapters_on)
        caches.append(c if keep else None)
    return h, caches, inputs


def stack_bwd(params, caches, shape, dh, adapters_on=True):
    grads = [None] * len(params["layers"])
    layer_dout = [None] * len(params["layers"])
    for li in range(len(params["layers"]) - 1, -1, -1):
        Wl, Ll = params["layers"][li]
        layer_dout[li] = dh
        dh, grads[li] = layer_bwd(caches[li], Wl, Ll, shape, dh, adapters_on)
    return grads, dh, layer_dout


def sft_step(params, ids, shape):
    """Mean next-token CE over B*(S-1) targets; returns (loss, grads, extras)."""
    h, caches, inputs = stack_fwd(params, ids, shape)
    logp, hc = token_logprobs(h, params["final_norm"], params["head"], ids, shape.eps)
    loss, dlogp = ce_loss(logp)
    dh = token_logprobs_bwd(hc, params["final_norm"], params["head"], ids, dlogp)
    grads, dh0, layer_dout = stack_bwd(params, caches, shape, dh)
    return loss, grads, dict(h_final=h, layer_inputs=inputs, layer_dout=layer_dout, dh_top=dh,
                             logp=logp)


def continuation_mask(S, prompt_len):
    """Target positions t (predicting token t+1) that lie in the continuation."""
    t = np.arange(S - 1)
    return (t + 1) >= prompt_len


def seq_logprob_sums(params, ids, shape, prompt_len, adapters_on):
    h, caches, _ = stack_fwd(params, ids, shape, adapters_on)
    logp, hc = token_logprobs(h, params["final_norm"], params["head"], ids, shape.eps)
    m = continuation_mask(ids.shape[1], prompt_len)
    return (logp * m[None, :]).sum(axis=1), (h, caches, hc, m)


def dpo_step(params, ids, shape, prompt_len, beta):
    """ids [2P, S]: rows 2p (chosen) and 2p+1 (rejected) share a prompt of
    ``prompt_len`` tokens.  Returns (loss, grads, extras)."""
    ref, _ = seq_logprob_sums(params, ids, shape, prompt_len, adapters_on=False)
    pol, (h, caches, hc, m) = seq_logprob_sums(params, ids, shape, prompt_len, adapters_on=True)
    loss, dc, dr = dpo_loss(pol[0::2], pol[1::2], ref[0::2], ref[1::2], beta)
    grads, ex = _policy_backward(params, ids, shape, (h, caches, hc, m), dc, dr)
    return loss, grads, dict(ex, policy=pol, reference=ref)


def _policy_backward(params, ids, shape, fwd, dc, dr):
    """Backward from dL/d(sequence sums) (chosen rows 2p, rejected 2p+1)
    through the continuation mask, the head and the stack."""
    h, caches, hc, m = fwd
    dseq = np.empty(ids.shape[0])
    dseq[0::2], dseq[1::2] = dc, dr
    dlogp = dseq[:, None] * m[None, :]
    dh = token_logprobs_bwd(hc, params["final_norm"], params["head"], ids, dlogp)
    grads, _, layer_dout = stack_bwd(params, caches, shape, dh)
    return grads, dict(dh_top=dh, layer_dout=layer_dout)


def simpo_step(params, ids, shape, prompt_len, beta, gamma):
    """Reference-free: one policy pass.  ids as for dpo_step; every row has
    S - prompt_len continuation targets."""
    pol, fwd = seq_logprob_sums(params, ids, shape, prompt_len, adapters_on=True)
    n = float(fwd[3].sum())
    loss, dc, dr = simpo_loss(pol[0::2], pol[1::2], n, n, beta, gamma)
    grads, ex = _policy_backward(params, ids, shape, fwd, dc, dr)
    return loss, grads, dict(ex, policy=pol)


def orpo_step(params, ids, shape, prompt_len, lam):
    pol, fwd = seq_logprob_sums(params, ids, shape, prompt_len, adapters_on=True)
    n = float(fwd[3].sum())
    loss, dc, dr = orpo_loss(pol[0::2], pol[1::2], n, n, lam)
    grads, ex = _policy_backward(params, ids, shape, fwd, dc, dr)
    return loss, grads, dict(ex, policy=pol)

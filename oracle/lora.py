"""LoRA linear layer over a frozen base weight (oracle; test infrastructure only).

Each adapted projection computes y = W x + s * B (A x) with s = alpha / r,
A [r, in], B [out, r] and the base W [out, in] frozen (LoRA as summarised on
the Soup pages: only the small adapters carry gradients and optimiser state,
"how layer streaming works"; and on the TRL/PEFT page, "LoRA with PEFT").
The backward pass follows the pages' remark that passing the gradient to the
layer below needs dL/dx = W^T dL/dy even though W is frozen: there is no dW.

Row-vector convention: x is [T, in] (one token per row), so the forward pass
is y = x W^T + s (x A^T) B^T.  fp64 throughout.

``adapters_on=False`` is the adapters-off model that DPO uses as its reference
(Soup pages, "memory-free reference model"; TRL/PEFT page, disabling the
adapter to get reference logits): the LoRA term is dropped entirely.
"""
from __future__ import annotations

import numpy as np


def lora_fwd(x, W, A, B, scale, adapters_on=True):
    """Returns (y [T, out], u [T, r]) with u = x A^T (unscaled)."""
    x = np.asarray(x, np.float64)
    W = np.asarray(W, np.float64)
    y = x @ W.T
    u = x @ np.asarray(A, np.float64).T
    if adapters_on:
        y = y + scale * (u @ np.asarray(B, np.float64).T)
    return y, u


def lora_bwd(x, W, A, B, scale, dy, adapters_on=True):
    """Gradients of a scalar loss given dL/dy [T, out].

    Returns (dx [T, in], dA [r, in], dB [out, r]); W gets no gradient.
      g  = dy B                (dL/d(s u) contracted with B)
      dx = dy W + s g A
      dA = s g^T x
      dB = s dy^T u,  u = x A^T
    """
    x = np.asarray(x, np.float64)
    W = np.asarray(W, np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    dy = np.asarray(dy, np.float64)
    dx = dy @ W
    if not adapters_on:
        return dx, np.zeros_like(A), np.zeros_like(B)
    g = dy @ B
    dx = dx + scale * (g @ A)
    dA = scale * (g.T @ x)
    dB = scale * (dy.T @ (x @ A.T))
    return dx, dA, dB

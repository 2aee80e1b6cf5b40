"""AdamW update of the LoRA adapters (oracle; test infrastructure only).

The Soup pages ("how layer streaming works") keep the LoRA adapters, their
gradients and the optimiser state resident in VRAM while the frozen base
streams; the pages' own run configures the learning rate (``lr: 5e-4``) and
nothing else about the optimiser.  The reading taken here is the default of
the Trainer the pages run on: AdamW with beta1 = 0.9, beta2 = 0.999,
eps = 1e-8, weight decay 0, fp32 parameters and fp32 moments.

AdamW is Adam with decoupled weight decay (Loshchilov & Hutter, "Decoupled
Weight Decay Regularization", ICLR 2019, the AdamW algorithm), written with a
fixed schedule multiplier and the decay folded into the learning rate
(lambda = lr * weight_decay), which is the parameterisation PyTorch and
transformers use.  For step t = 1, 2, ...:

    g     = grad_scale * grad
    theta = theta - lr * weight_decay * theta          (decay on the old theta)
    m     = beta1 * m + (1 - beta1) * g
    v     = beta2 * v + (1 - beta2) * g^2
    m_hat = m / (1 - beta1^t)
    v_hat = v / (1 - beta2^t)
    theta = theta - lr * m_hat / (sqrt(v_hat) + eps)

``grad_scale`` multiplies the incoming gradient (1 / world size when the
gradient arrives as a data-parallel sum).  fp64 throughout: the fp32
parameters and moments a caller holds are exact fp64 numbers.
"""
from __future__ import annotations

import numpy as np


def adamw_step(theta, grad, m, v, t, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, grad_scale=1.0):
    """One AdamW step.  Returns (theta, m, v) as new fp64 arrays; t >= 1 is
    the index of this step (the bias corrections use beta^t)."""
    if t < 1:
        raise ValueError("step index t starts at 1")
    theta = np.array(theta, np.float64)
    g = np.asarray(grad, np.float64) * grad_scale
    m = np.asarray(m, np.float64)
    v = np.asarray(v, np.float64)
    theta = theta - lr * weight_decay * theta
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** t)
    v_hat = v / (1.0 - beta2 ** t)
    theta = theta - lr * m_hat / (np.sqrt(v_hat) + eps)
    return theta, m, v


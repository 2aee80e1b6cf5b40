"""One Llama-style decoder layer with LoRA on all seven projections
(oracle; test infrastructure only).

The pages stream "one decoder layer at a time" (Soup pages, "layer
streaming"), but do not spell out the layer.  The layer is the Llama-3.1-8B /
Qwen2.5 shape of the workloads:

  x1  = RMSNorm(h; w1)
  q, k, v = LoRA projections of x1;  q, k rotated by RoPE
  att = causal GQA attention(q, k, v)
  h2  = h + LoRA_o(att)
  x2  = RMSNorm(h2; w2)
  a   = silu(LoRA_gate(x2)) * LoRA_up(x2)
  out = h2 + LoRA_down(a)

Readings (where the pages are silent): RMSNorm
y = x / sqrt(mean(x^2) + eps) * w with frozen w; RoPE is the rotate-half form
pairing (i, i + d/2) with inv_freq_i = theta^(-2i/d), no frequency rescaling,
positions restarting at 0 in every sequence; attention scale 1/sqrt(d), causal
within a sequence, kv head = q_head // (Hq / Hkv); no biases; no dropout.

The backward pass is the chain rule written out by hand per operation, in
fp64, for the recompute-style backward of the pages ("how layer streaming
works": the layer is re-read and recomputed, and the gradient to the layer
below is dL/dx = W^T dL/dy plus the adapter terms; W gets no gradient).
"""
from __future__ import annotations

import numpy as np

from .lora import lora_bwd, lora_fwd

PROJS = ("q", "k", "v", "o", "gate", "up", "down")


# ----------------------------------------------------------------------------- RMSNorm
def rmsnorm_fwd(x, w, eps):
    x = np.asarray(x, np.float64)
    rinv = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * rinv * np.asarray(w, np.float64), rinv


def rmsnorm_bwd(x, w, rinv, dy):
    """dL/dx of y = x * rinv(x) * w (w frozen)."""
    x = np.asarray(x, np.float64)
    xh = x * rinv
    dxh = np.asarray(dy, np.float64) * np.asarray(w, np.float64)
    return rinv * (dxh - xh * np.mean(dxh * xh, axis=-1, keepdims=True))


# ----------------------------------------------------------------------------- RoPE
def rope_tables(S, head_dim, theta):
    half = head_dim // 2
    inv = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / head_dim)
    ang = np.arange(S, dtype=np.float64)[:, None] * inv[None, :]
    return np.cos(ang), np.sin(ang)          # [S, half]


def rope_fwd(t, cos, sin):
    """t [B, S, nh, d]: rotate pairs (i, i + d/2) by the position's angle."""
    half = t.shape[-1] // 2
    t1, t2 = t[..., :half], t[..., half:]
    c, s = cos[None, :, None, :], sin[None, :, None, :]
    return np.concatenate([t1 * c - t2 * s, t2 * c + t1 * s], axis=-1)


def rope_bwd(dt, cos, sin):
    """Transpose of the rotation (rotate by the negative angle)."""
    half = dt.shape[-1] // 2
    d1, d2 = dt[..., :half], dt[..., half:]
    c, s = cos[None, :, None, :], sin[None, :, None, :]
    return np.concatenate([d1 * c + d2 * s, d2 * c - d1 * s], axis=-1)


# ----------------------------------------------------------------------------- attention
def attention_fwd(q, k, v):
    """q [B,S,Hq,d], k/v [B,S,Hkv,d] -> (out [B,S,Hq,d], P list per (b, h))."""
    Bsz, S, Hq, d = q.shape
    Hkv = k.shape[2]
    grp = Hq // Hkv
    scale = 1.0 / np.sqrt(d)
    mask = np.triu(np.ones((S, S), dtype=bool), k=1)
    out = np.empty_like(q)
    probs = {}
    for b in range(Bsz):
        for h in range(Hq):
            g = h // grp
            sc = (q[b, :, h, :] @ k[b, :, g, :].T) * scale
            sc[mask] = -np.inf
            m = sc.max(axis=1, keepdims=True)
            e = np.exp(sc - m)
            P = e / e.sum(axis=1, keepdims=True)
            out[b, :, h, :] = P @ v[b, :, g, :]
            probs[(b, h)] = P
    return out, probs


def attention_bwd(q, k, v, probs, dout):
    Bsz, S, Hq, d = q.shape
    Hkv = k.shape[2]
    grp = Hq // Hkv
    scale = 1.0 / np.sqrt(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(Bsz):
        for h in range(Hq):
            g = h // grp
            P = probs[(b, h)]
            do = dout[b, :, h, :]
            dv[b, :, g, :] += P.T @ do
            dP = do @ v[b, :, g, :].T
            dS = P * (dP - np.sum(dP * P, axis=1, keepdims=True))
            dq[b, :, h, :] = (dS @ k[b, :, g, :]) * scale
            dk[b, :, g, :] += (dS.T @ q[b, :, h, :]) * scale
    return dq, dk, dv


# ----------------------------------------------------------------------------- SwiGLU
def _sigmoid(x):
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def swiglu_fwd(g, u):
    return g * _sigmoid(g) * u


def swiglu_bwd(g, u, da):
    sg = _sigmoid(g)
    silu = g * sg
    dg = da * u * sg * (1.0 + g * (1.0 - sg))
    du = da * silu
    return dg, du


# ----------------------------------------------------------------------------- the layer
def _proj(x2d, Wd, lora, p, s, on):
    A, B = lora[p]
    return lora_fwd(x2d, Wd[p], A, B, s, on)[0]


def layer_fwd(h, W, lora, shape, adapters_on=True):
    """h [B, S, H] -> (h_out [B, S, H], cache).

    W: dict proj -> dequantised base weight [out, in] plus 'norm1', 'norm2'.
    lora: dict proj -> (A [r, in], B [out, r]).
    """
    h = np.asarray(h, np.float64)
    Bsz, S, H = h.shape
    Hq, Hkv, d = shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    s = shape.alpha / shape.rank
    T = Bsz * S
    x1, r1 = rmsnorm_fwd(h, W["norm1"], shape.eps)
    x1f = x1.reshape(T, H)
    q = _proj(x1f, W, lora, "q", s, adapters_on).reshape(Bsz, S, Hq, d)
    k = _proj(x1f, W, lora, "k", s, adapters_on).reshape(Bsz, S, Hkv, d)
    v = _proj(x1f, W, lora, "v", s, adapters_on).reshape(Bsz, S, Hkv, d)
    cos, sin = rope_tables(S, d, shape.theta)
    qr = rope_fwd(q, cos, sin)
    kr = rope_fwd(k, cos, sin)
    att, probs = attention_fwd(qr, kr, v)
    attf = att.reshape(T, Hq * d)
    o = _proj(attf, W, lora, "o", s, adapters_on).reshape(Bsz, S, H)
    h2 = h + o
    x2, r2 = rmsnorm_fwd(h2, W["norm2"], shape.eps)
    x2f = x2.reshape(T, H)
    g = _proj(x2f, W, lora, "gate", s, adapters_on)
    u = _proj(x2f, W, lora, "up", s, adapters_on)
    a = swiglu_fwd(g, u)
    dn = _proj(a, W, lora, "down", s, adapters_on).reshape(Bsz, S, H)
    out = h2 + dn
    cache = dict(h=h, x1=x1f, r1=r1, qr=qr, kr=kr, v=v, probs=probs, cos=cos, sin=sin,
                 attf=attf, h2=h2, x2=x2f, r2=r2, g=g, u=u, a=a)
    return out, cache


def layer_bwd(cache, W, lora, shape, dout, adapters_on=True):
    """Backward of ``layer_fwd``.  Returns (dh_in [B,S,H], grads) with
    grads: proj -> (dA [r, in], dB [out, r])."""
    dout = np.asarray(dout, np.float64)
    Bsz, S, H = dout.shape
    Hq, Hkv, d = shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    s = shape.alpha / shape.rank
    T = Bsz * S
    grads = {}

    def back(p, x, dy):
        A, B = lora[p]
        dx, dA, dB = lora_bwd(x, W[p], A, B, s, dy, adapters_on)
        grads[p] = (dA, dB)
        return dx

    # MLP block: out = h2 + down(swiglu(gate(x2), up(x2)))
    dd = dout.reshape(T, H)
    da = back("down", cache["a"], dd)
    dg, du = swiglu_bwd(cache["g"], cache["u"], da)
    dx2 = back("gate", cache["x2"], dg) + back("up", cache["x2"], du)
    dh2 = dout + rmsnorm_bwd(cache["h2"], W["norm2"], cache["r2"], dx2.reshape(Bsz, S, H))

    # attention block: h2 = h + o(attn(rope(q(x1)), rope(k(x1)), v(x1)))
    datt = back("o", cache["attf"], dh2.reshape(T, H)).reshape(Bsz, S, Hq, d)
    dqr, dkr, dv = attention_bwd(cache["qr"], cache["kr"], cache["v"], cache["probs"], datt)
    dq = rope_bwd(dqr, cache["cos"], cache["sin"])
    dk = rope_bwd(dkr, cache["cos"], cache["sin"])
    x1 = cache["x1"]
    dx1 = (back("q", x1, dq.reshape(T, Hq * d)) + back("k", x1, dk.reshape(T, Hkv * d))
           + back("v", x1, dv.reshape(T, Hkv * d)))
    dh = dh2 + rmsnorm_bwd(cache["h"], W["norm1"], cache["r1"], dx1.reshape(Bsz, S, H))
    return dh, grads

"""Pins for the decoder-layer oracle (CPU): directional finite differences of
every gradient, attention special cases with closed forms (one token, zero
queries), causality, RoPE invariants, RMSNorm of a constant row, GQA as
duplicated kv heads, and the B = 0 / adapters-off identities."""
import numpy as np
import pytest

import soup_synth as ss
from oracle import layer as L
from oracle.layer import layer_bwd, layer_fwd

PROJS = ss.PROJ_NAMES


def _params(shape, seed=0, zero_B=False, wscale=0.2):
    g = np.random.default_rng(seed)
    W = {p: g.standard_normal(shape.proj_shape(p)) * wscale for p in PROJS}
    W["norm1"] = 1 + 0.1 * g.standard_normal(shape.hidden)
    W["norm2"] = 1 + 0.1 * g.standard_normal(shape.hidden)
    lora = {}
    for p in PROJS:
        o, i = shape.proj_shape(p)
        A = g.standard_normal((shape.rank, i)) * 0.3
        B = np.zeros((o, shape.rank)) if zero_B else g.standard_normal((o, shape.rank)) * 0.3
        lora[p] = (A, B)
    return W, lora


SHAPE = ss.tiny_layer_shape(hidden=16, n_q=4, n_kv=2, head_dim=4, inter=24, rank=2, alpha=4.0)


def test_layer_directional_finite_differences():
    shape = SHAPE
    W, lora = _params(shape, seed=1)
    g = np.random.default_rng(2)
    h = g.standard_normal((2, 5, shape.hidden))
    R = g.standard_normal(h.shape)
    obj = lambda h_, lora_: float(np.sum(layer_fwd(h_, W, lora_, shape)[0] * R))
    out, cache = layer_fwd(h, W, lora, shape)
    dh, grads = layer_bwd(cache, W, lora, shape, R)
    eps = 1e-6
    for trial in range(3):
        v = g.standard_normal(h.shape)
        num = (obj(h + eps * v, lora) - obj(h - eps * v, lora)) / (2 * eps)
        ana = float(np.sum(dh * v))
        assert abs(num - ana) <= 1e-6 * max(1.0, abs(ana)), (num, ana)
    for p in PROJS:
        for which in (0, 1):
            base = lora[p][which]
            v = g.standard_normal(base.shape)
            lp = dict(lora); lm = dict(lora)
            pair_p, pair_m = list(lora[p]), list(lora[p])
            pair_p[which] = base + eps * v
            pair_m[which] = base - eps * v
            lp[p], lm[p] = tuple(pair_p), tuple(pair_m)
            num = (obj(h, lp) - obj(h, lm)) / (2 * eps)
            ana = float(np.sum(grads[p][which] * v))
            assert abs(num - ana) <= 1e-6 * max(1.0, abs(ana)), (p, which, num, ana)


def test_attention_single_token_returns_v():
    g = np.random.default_rng(0)
    q = g.standard_normal((2, 1, 4, 8)); k = g.standard_normal((2, 1, 2, 8)); v = g.standard_normal((2, 1, 2, 8))
    out, _ = L.attention_fwd(q, k, v)
    for h in range(4):
        assert np.array_equal(out[:, :, h, :], v[:, :, h // 2, :])


def test_attention_zero_queries_is_prefix_mean():
    g = np.random.default_rng(1)
    S = 6
    q = np.zeros((1, S, 2, 4)); k = g.standard_normal((1, S, 1, 4)); v = g.standard_normal((1, S, 1, 4))
    out, _ = L.attention_fwd(q, k, v)
    for i in range(S):
        np.testing.assert_allclose(out[0, i, 0], v[0, :i + 1, 0].mean(axis=0), rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(out[0, i, 1], v[0, :i + 1, 0].mean(axis=0), rtol=1e-13, atol=1e-13)


def test_layer_is_causal():
    shape = SHAPE
    W, lora = _params(shape, seed=3)
    g = np.random.default_rng(4)
    h = g.standard_normal((1, 7, shape.hidden))
    base, _ = layer_fwd(h, W, lora, shape)
    h2 = h.copy(); h2[0, 4] += 1.0
    pert, _ = layer_fwd(h2, W, lora, shape)
    assert np.array_equal(base[0, :4], pert[0, :4])
    assert not np.allclose(base[0, 4:], pert[0, 4:])


def test_rope_invariants():
    g = np.random.default_rng(5)
    S, d = 9, 8
    cos, sin = L.rope_tables(S, d, 5e5)
    t = g.standard_normal((1, S, 3, d))
    r = L.rope_fwd(t, cos, sin)
    assert np.array_equal(r[:, 0], t[:, 0])                    # position 0 is the identity
    half = d // 2
    n0 = t[..., :half] ** 2 + t[..., half:] ** 2
    n1 = r[..., :half] ** 2 + r[..., half:] ** 2
    np.testing.assert_allclose(n1, n0, rtol=1e-12)             # each pair keeps its norm
    np.testing.assert_allclose(L.rope_bwd(r, cos, sin), t, rtol=1e-12, atol=1e-12)  # inverse
    # relative-position property: <R_m q, R_n k> depends on m - n only
    q = g.standard_normal(d); k = g.standard_normal(d)
    Q = L.rope_fwd(np.broadcast_to(q, (1, S, 1, d)).copy(), cos, sin)[0, :, 0]
    K = L.rope_fwd(np.broadcast_to(k, (1, S, 1, d)).copy(), cos, sin)[0, :, 0]
    np.testing.assert_allclose(Q[5] @ K[2], Q[7] @ K[4], rtol=1e-9)
    np.testing.assert_allclose(Q[3] @ K[3], q @ k, rtol=1e-9)


def test_rmsnorm_constant_row_is_sign_times_weight():
    w = np.array([0.5, 2.0, -1.5, 1.0])
    x = np.array([[0.25] * 4, [-8.0] * 4])
    y, _ = L.rmsnorm_fwd(x, w, 0.0)
    assert np.array_equal(y[0], w) and np.array_equal(y[1], -w)


def test_swiglu_special_values():
    g = np.array([0.0, 40.0, -40.0]); u = np.array([3.0, 2.0, 5.0])
    a = L.swiglu_fwd(g, u)
    assert a[0] == 0.0
    np.testing.assert_allclose(a[1], 80.0, rtol=1e-15)
    assert abs(a[2]) < 1e-15
    dg, du = L.swiglu_bwd(np.array([0.0]), np.array([3.0]), np.array([1.0]))
    assert dg[0] == 1.5 and du[0] == 0.0                       # silu'(0) = 1/2


def test_gqa_equals_duplicated_kv_heads():
    s_gqa = ss.tiny_layer_shape(hidden=16, n_q=4, n_kv=2, head_dim=4, inter=24, rank=2)
    s_mha = ss.tiny_layer_shape(hidden=16, n_q=4, n_kv=4, head_dim=4, inter=24, rank=2)
    W, lora = _params(s_gqa, seed=6)
    W2, lora2 = dict(W), dict(lora)
    d = 4
    for p in ("k", "v"):
        w = W[p].reshape(2, d, 16)
        W2[p] = np.repeat(w, 2, axis=0).reshape(16, 16)
        A, B = lora[p]
        B2 = np.repeat(B.reshape(2, d, 2), 2, axis=0).reshape(16, 2)
        lora2[p] = (A, B2)
    h = np.random.default_rng(7).standard_normal((1, 5, 16))
    o1, _ = layer_fwd(h, W, lora, s_gqa)
    o2, _ = layer_fwd(h, W2, lora2, s_mha)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-12)


def test_B_zero_and_adapters_off_reproduce_base_exactly():
    shape = SHAPE
    W, lora = _params(shape, seed=8)
    _, lora0 = _params(shape, seed=8, zero_B=True)
    h = np.random.default_rng(9).standard_normal((2, 4, shape.hidden))
    off, _ = layer_fwd(h, W, lora, shape, adapters_on=False)
    zero, _ = layer_fwd(h, W, lora0, shape)
    assert np.array_equal(off, zero)
    on, _ = layer_fwd(h, W, lora, shape)
    assert not np.allclose(on, off)


# ----------------------------------------------------------------------------- constants pinned by closed forms
# Each test below fails if the oracle's RoPE exponent, attention scale or
# RMSNorm epsilon placement is changed: the expected values are computed from
# scalar closed forms (math module), not by re-running the oracle's formula.
import math


def test_rope_frequencies_at_position_one_closed_form():
    """The 8B layer (theta 5e5, head_dim 128): at position 1, pair i turns by
    exactly theta^(-2i/128) radians, so pair 0 turns by 1 rad and the last
    pair (i = 63) by 5e5^(-126/128).  A rotated unit vector e_i reads
    (cos a_i, sin a_i) in components (i, i + 64)."""
    d, theta = 128, 5e5
    assert ss.LLAMA8B_LAYER.theta == 5e5 and ss.LLAMA8B_LAYER.head_dim == d
    cos, sin = L.rope_tables(2, d, theta)
    for i, angle in ((0, 1.0), (32, 5e5 ** -0.5), (63, 5e5 ** (-126.0 / 128.0))):
        e = np.zeros((1, 2, 1, d))
        e[0, 1, 0, i] = 1.0
        r = L.rope_fwd(e, cos, sin)[0, 1, 0]
        assert abs(r[i] - math.cos(angle)) < 1e-15, (i, r[i], math.cos(angle))
        assert abs(r[i + 64] - math.sin(angle)) < 1e-15, (i, r[i + 64], math.sin(angle))
        others = np.delete(r, [i, i + 64])
        assert np.all(others == 0.0)
    # the second component of a pair turns the other way: e_{i+64} -> (-sin a, cos a)
    e = np.zeros((1, 2, 1, d))
    e[0, 1, 0, 64] = 1.0
    r = L.rope_fwd(e, cos, sin)[0, 1, 0]
    assert abs(r[0] + math.sin(1.0)) < 1e-15 and abs(r[64] - math.cos(1.0)) < 1e-15
    # position p turns pair 0 by p rad (not p * anything else)
    cos7, sin7 = L.rope_tables(8, d, theta)
    assert abs(cos7[7, 0] - math.cos(7.0)) < 1e-15 and abs(sin7[7, 0] - math.sin(7.0)) < 1e-15


def test_attention_scale_two_token_closed_form():
    """head_dim 128, two tokens with k0 = 0 and q1 . k1 = c: the second query's
    softmax weights are 1 / (1 + e^(c/sqrt(128))) on v0 and
    e^(c/sqrt(128)) / (1 + e^(c/sqrt(128))) on v1."""
    d, c = 128, 3.0
    g = np.random.default_rng(11)
    q = np.zeros((1, 2, 1, d)); k = np.zeros((1, 2, 1, d)); v = np.zeros((1, 2, 1, d))
    q[0, 1, 0] = g.standard_normal(d)
    k1 = g.standard_normal(d)
    k1 *= c / float(q[0, 1, 0] @ k1)               # q1 . k1 = c exactly up to rounding
    k[0, 1, 0] = k1
    v[0, 0, 0, 0] = 1.0                            # v0 = e_0, v1 = e_1
    v[0, 1, 0, 1] = 1.0
    out, _ = L.attention_fwd(q, k, v)
    z = math.exp(c / math.sqrt(128.0))
    assert abs(out[0, 1, 0, 0] - 1.0 / (1.0 + z)) < 1e-13
    assert abs(out[0, 1, 0, 1] - z / (1.0 + z)) < 1e-13
    assert np.all(out[0, 1, 0, 2:] == 0.0)


def test_rmsnorm_eps_inside_the_root_constant_row():
    """A constant row c with eps > 0 normalises to w * c / sqrt(c^2 + eps)
    (eps added to the mean square, inside the square root)."""
    eps = 1e-5
    w = np.array([0.5, 2.0, -1.5, 1.0])
    for c in (0.01, -0.003, 2.0):
        x = np.full((1, 4), c)
        y, rinv = L.rmsnorm_fwd(x, w, eps)
        expect = c / math.sqrt(c * c + eps)
        np.testing.assert_allclose(y[0], w * expect, rtol=1e-14, atol=0)
        assert abs(rinv[0, 0] - 1.0 / math.sqrt(c * c + eps)) <= 1e-14 / math.sqrt(c * c + eps)
    assert ss.LLAMA8B_LAYER.eps == 1e-5

"""The causal GQA attention kernels (tcgen05, accumulators in tensor memory)
through the C ABI against the oracle's attention (fp64, plain softmax):
output, log-sum-exp, dq, dk, dv within relative Frobenius 5e-3 and
max|diff| 1e-2 max|ref|, on shapes that span several 128-row tiles with
ragged tails, a one-token sequence, GQA groups of 1, 2 and 4, and several
sequences per batch.  The inputs are fp16-exact, so both sides see the same
numbers; the backward is deterministic (same bits twice)."""
import numpy as np
import pytest
import torch

import soup_synth as ss
from oracle import layer as OL
from tests.gpu_util import assert_close, host

pytestmark = pytest.mark.gpu
HD = 128


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from layer_streamed_qlora_b200 import _lib as lib
    lib.lib()
    yield lib
    assert lib.device_error() == 0


def f16_values(a):
    return np.asarray(a, np.float32).astype(np.float16).astype(np.float64)


def run_case(L, B, S, Hq, Hkv, seed, qscale=1.0, pad_cols=0):
    T = B * S
    ld = (Hq + 2 * Hkv) * HD + pad_cols
    qkv = f16_values(ss.normal_f32(seed, "attn.qkv", (T, ld)) * np.float32(qscale))
    dout = f16_values(ss.normal_f32(seed, "attn.dout", (T, Hq * HD)))
    qkv_d = torch.from_numpy(qkv.astype(np.float16)).cuda()
    dout_d = torch.from_numpy(dout.astype(np.float16)).cuda()
    out = torch.empty((T, Hq * HD), dtype=torch.bfloat16, device="cuda")
    out16 = torch.empty((T, Hq * HD), dtype=torch.float16, device="cuda")
    lse = torch.empty((Hq, T), dtype=torch.float32, device="cuda")
    L.soup_attention_fwd(qkv_d, B, S, Hq, Hkv, out, out16, lse)
    D = torch.empty((Hq, T), dtype=torch.float32, device="cuda")
    dqkv = torch.zeros((T, ld), dtype=torch.bfloat16, device="cuda")
    dqkv32 = torch.zeros((T, ld), dtype=torch.float32, device="cuda")
    L.soup_attention_bwd(qkv_d, B, S, Hq, Hkv, out16, dout_d, lse, D, dqkv, dqkv32)
    torch.cuda.synchronize()
    got = dict(out=host(out), lse=host(lse), dqkv=host(dqkv), dqkv32=host(dqkv32))
    # oracle on the same fp16-exact values
    q = qkv[:, :Hq * HD].reshape(B, S, Hq, HD)
    k = qkv[:, Hq * HD:(Hq + Hkv) * HD].reshape(B, S, Hkv, HD)
    v = qkv[:, (Hq + Hkv) * HD:(Hq + 2 * Hkv) * HD].reshape(B, S, Hkv, HD)
    ref, probs = OL.attention_fwd(q, k, v)
    dq, dk, dv = OL.attention_bwd(q, k, v, probs, dout.reshape(B, S, Hq, HD))
    # log2 of each row's softmax denominator (with the row maximum)
    sc = 1.0 / np.sqrt(HD)
    lse_ref = np.empty((Hq, T))
    for b in range(B):
        for h in range(Hq):
            z = (q[b, :, h] @ k[b, :, h // (Hq // Hkv)].T) * sc
            z[np.triu(np.ones((S, S), bool), 1)] = -np.inf
            mx = z.max(axis=1)
            lse_ref[h, b * S:(b + 1) * S] = (mx + np.log(np.exp(z - mx[:, None]).sum(axis=1))) / np.log(2.0)
    return got, dict(out=ref.reshape(T, Hq * HD), lse=lse_ref, dq=dq.reshape(T, -1), dk=dk.reshape(T, -1),
                     dv=dv.reshape(T, -1)), (qkv_d, dout_d, out16, lse, D, dqkv, ld)


CASES = [
    (2, 100, 4, 2),    # ragged single tile per sequence, GQA group 2
    (1, 256, 4, 1),    # two full tiles, one kv head for four q heads
    (3, 130, 8, 2),    # a full tile and a 2-row tail, three sequences
    (1, 1, 2, 2),      # one token: the output is v
    (2, 384, 2, 2),    # three tiles, no grouping
    (1, 517, 8, 2),    # five tiles with a 5-row tail
]


@pytest.mark.parametrize("B,S,Hq,Hkv", CASES)
def test_attention_matches_oracle(L, B, S, Hq, Hkv):
    got, ref, _ = run_case(L, B, S, Hq, Hkv, seed=B * 1000 + S)
    assert_close(got["out"], ref["out"], f"out B{B} S{S}")
    assert np.max(np.abs(got["lse"] - ref["lse"])) < 2e-3, np.max(np.abs(got["lse"] - ref["lse"]))
    qo, ko = Hq * HD, (Hq + Hkv) * HD
    for name, g32, gbf in (("dq", got["dqkv32"][:, :qo], got["dqkv"][:, :qo]),
                           ("dk", got["dqkv32"][:, qo:ko], got["dqkv"][:, qo:ko]),
                           ("dv", got["dqkv32"][:, ko:ko + Hkv * HD], got["dqkv"][:, ko:ko + Hkv * HD])):
        if not np.any(ref[name]):
            # one token: the softmax is the constant 1, so dq = dk = 0 exactly;
            # the kernel's dP - D cancels to rounding level (D comes from the
            # fp16 output, dP from the MMA)
            assert np.max(np.abs(g32)) < 1e-5 and np.max(np.abs(gbf)) < 1e-5, name
            continue
        assert_close(g32, ref[name], f"{name} (fp32) B{B} S{S}")
        assert_close(gbf, ref[name], f"{name} (bf16) B{B} S{S}")


def test_attention_large_logits_and_row_stride(L):
    """q, k scaled x4 (logits ~16x sharper) and a row stride with 8 extra
    columns: the same tolerances hold and the extra columns stay untouched."""
    got, ref, _ = run_case(L, 2, 200, 4, 2, seed=77, qscale=2.0, pad_cols=8)
    assert_close(got["out"], ref["out"], "out (sharp)")
    qo = 4 * HD
    assert_close(got["dqkv32"][:, :qo], ref["dq"], "dq (sharp)")
    assert np.all(got["dqkv"][:, -8:] == 0.0)


def test_attention_backward_is_deterministic(L):
    got, _, (qkv_d, dout_d, out16, lse, D, dqkv, ld) = run_case(L, 2, 300, 8, 2, seed=5)
    first = dqkv.clone()
    L.soup_attention_bwd(qkv_d, 2, 300, 8, 2, out16, dout_d, lse, D, dqkv)
    torch.cuda.synchronize()
    assert torch.equal(first, dqkv)


def test_attention_with_a_shared_prefix_matches_oracle(L):
    """Two groups of G = 2 sequences (preference pairs) sharing a 256-token
    prefix stored once, with 100-token continuations (ragged): each
    sequence's output equals the oracle's attention over that sequence
    expanded (prefix + its own continuation); the prefix's gradients sum the
    contributions of both sequences of its group (its queries belong to the
    group's first sequence, whose output the prefix rows hold)."""
    G, P, Lp, Lc, Hq, Hkv = 2, 2, 256, 100, 8, 2
    S = Lp + Lc
    span = Lp + G * Lc
    T = P * span
    ld = (Hq + 2 * Hkv) * HD
    qkv = f16_values(ss.normal_f32(31, "attn.share.qkv", (T, ld)))
    dout = f16_values(ss.normal_f32(31, "attn.share.dout", (T, Hq * HD)))
    qkv_d = torch.from_numpy(qkv.astype(np.float16)).cuda()
    dout_d = torch.from_numpy(dout.astype(np.float16)).cuda()
    out = torch.empty((T, Hq * HD), dtype=torch.bfloat16, device="cuda")
    out16 = torch.empty((T, Hq * HD), dtype=torch.float16, device="cuda")
    lse = torch.empty((Hq, T), dtype=torch.float32, device="cuda")
    L.soup_attention_fwd(qkv_d, P * G, S, Hq, Hkv, out, out16, lse, prefix_share=G, prefix_len=Lp)
    D = torch.empty((Hq, T), dtype=torch.float32, device="cuda")
    dqkv32 = torch.zeros((T, ld), dtype=torch.float32, device="cuda")
    dqkv = torch.zeros((T, ld), dtype=torch.bfloat16, device="cuda")
    L.soup_attention_bwd(qkv_d, P * G, S, Hq, Hkv, out16, dout_d, lse, D, dqkv, dqkv32, prefix_share=G, prefix_len=Lp)
    torch.cuda.synchronize()
    got_out, got_d = host(out), host(dqkv32)
    ref_out = np.zeros((T, Hq * HD))
    ref_d = np.zeros((T, ld))
    for p in range(P):
        base = p * span
        for i in range(G):
            rows = np.concatenate([np.arange(base, base + Lp), np.arange(base + Lp + i * Lc, base + Lp + (i + 1) * Lc)])
            x = qkv[rows]
            q = x[:, :Hq * HD].reshape(1, S, Hq, HD)
            k = x[:, Hq * HD:(Hq + Hkv) * HD].reshape(1, S, Hkv, HD)
            v = x[:, (Hq + Hkv) * HD:(Hq + 2 * Hkv) * HD].reshape(1, S, Hkv, HD)
            o, probs = OL.attention_fwd(q, k, v)
            do = dout[rows].copy()
            if i > 0:
                do[:Lp] = 0.0  # the prefix's outputs are the first sequence's
            dq, dk, dv = OL.attention_bwd(q, k, v, probs, do.reshape(1, S, Hq, HD))
            own = rows if i == 0 else rows[Lp:]
            sl = slice(0, S) if i == 0 else slice(Lp, S)
            ref_out[own] = o.reshape(S, -1)[sl]
            grads = np.concatenate([dq.reshape(S, -1), dk.reshape(S, -1), dv.reshape(S, -1)], axis=1)
            ref_d[rows] += grads  # prefix rows: dk, dv from every sequence (dq of a later one is 0)
    assert_close(got_out, ref_out, "out (shared prefix)")
    qo, ko = Hq * HD, (Hq + Hkv) * HD
    assert_close(got_d[:, :qo], ref_d[:, :qo], "dq (shared prefix)")
    assert_close(got_d[:, qo:ko], ref_d[:, qo:ko], "dk (shared prefix)")
    assert_close(got_d[:, ko:], ref_d[:, ko:], "dv (shared prefix)")


def test_attention_16_byte_output_fallback_bit_exact(L):
    """Outputs 16- but not 32-byte aligned take the epilogues' 16-byte stores
    instead of their 32-byte ones: the same bits either way."""
    B, S, Hq, Hkv = 3, 130, 8, 2
    got, _, (qkv_d, dout_d, out16, lse, D, dqkv, ld) = run_case(L, B, S, Hq, Hkv, seed=21)
    T = B * S

    def offset_view(shape, dtype):
        n = shape[0] * shape[1]
        buf = torch.zeros(n + 32 // torch.tensor([], dtype=dtype).element_size(), dtype=dtype, device="cuda")
        v = buf[16 // buf.element_size():16 // buf.element_size() + n].view(*shape)
        assert v.data_ptr() % 32 == 16
        return v

    out = offset_view((T, Hq * HD), torch.bfloat16)
    o16 = offset_view((T, Hq * HD), torch.float16)
    lse2 = torch.empty((Hq, T), dtype=torch.float32, device="cuda")
    L.soup_attention_fwd(qkv_d, B, S, Hq, Hkv, out, o16, lse2)
    dq2 = offset_view((T, ld), torch.bfloat16)
    dq32 = offset_view((T, ld), torch.float32)
    D2 = torch.empty((Hq, T), dtype=torch.float32, device="cuda")
    L.soup_attention_bwd(qkv_d, B, S, Hq, Hkv, o16, dout_d, lse2, D2, dq2, dq32)
    torch.cuda.synchronize()
    assert np.array_equal(host(out), got["out"])
    assert np.array_equal(host(lse2), got["lse"])
    assert np.array_equal(host(dq2), got["dqkv"])
    assert np.array_equal(host(dq32), got["dqkv32"])

"""GPU parity of the NF4 kernels and of one LoRA-adapted projection against
the CPU oracle, through the C ABI.

* NF4 codes, absmax and dequantised bf16 weights: bit-exact.
* LoRA linear forward/backward (y, u, dx, dA, dB): relative Frobenius error
  <= 5e-3 and max |diff| <= 1e-2 max |ref|.
* The fused NF4-decode GEMM equals "dequantise, then bf16 GEMM" bit for bit,
  and B = 0 reproduces the frozen-base output exactly.
"""
import numpy as np
import pytest
import torch

import soup_synth as ss
from oracle import nf4 as onf4
from oracle.lora import lora_bwd, lora_fwd
from tests.gpu_util import assert_close, dev_bf16, dev_f32, host

pytestmark = pytest.mark.gpu

L = None


@pytest.fixture(scope="module", autouse=True)
def _lib():
    global L
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from layer_streamed_qlora_b200 import _lib as lib
    lib.lib()
    L = lib
    yield
    assert lib.device_error() == 0


def gpu_quantize(W32):
    out_f, in_f = W32.shape
    W = dev_f32(W32)
    codes = torch.empty((out_f, in_f // 2), dtype=torch.uint8, device="cuda")
    absmax = torch.empty((out_f, in_f // 64), dtype=torch.float32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.soup_nf4_quantize(W, codes, absmax, flag)
    return codes, absmax


def gpu_dequant(codes, absmax, out_f, in_f):
    Wb = torch.empty((out_f, in_f), dtype=torch.bfloat16, device="cuda")
    L.soup_nf4_dequant(codes, absmax, out_f, in_f, Wb)
    return Wb


@pytest.mark.parametrize("shape", [(512, 512), (48, 128), (4096, 256)])
def test_nf4_quantize_dequant_bit_exact(shape):
    W = ss.normal_f32(0, f"nf4.{shape}", shape, std=0.02)
    W[0, :64] = 0.0                                   # all-zero block
    W[1, 5] = 0.0
    codes, absmax = gpu_quantize(W)
    oc, oa = onf4.quantize(W)
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(absmax.cpu().numpy().view(np.uint32), oa.view(np.uint32))
    Wb = gpu_dequant(codes, absmax, *shape)
    od = onf4.dequant_bf16(oc, oa)
    assert np.array_equal(Wb.float().cpu().numpy().view(np.uint32), od.view(np.uint32))


def test_nf4_midpoint_ties_and_extremes_bit_exact():
    cb = onf4.NF4_CODEBOOK.astype(np.float64)
    W = np.zeros((2, 128), np.float32)
    W[0, 0] = 1.0
    j = 1
    for i in range(15):
        m = 0.5 * (cb[i] + cb[i + 1])
        f = np.float32(m)
        W[0, j] = f                                   # near/at midpoint
        W[0, j + 1] = np.nextafter(f, np.float32(2))
        W[0, j + 2] = np.nextafter(f, np.float32(-2))
        j += 3
    W[1, :] = np.linspace(-3, 3, 128, dtype=np.float32)
    codes, absmax = gpu_quantize(W)
    oc, oa = onf4.quantize(W)
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(absmax.cpu().numpy(), oa)


def test_nf4_nonfinite_refused():
    W = np.zeros((4, 64), np.float32)
    W[2, 3] = np.inf
    with pytest.raises(L.SoupError) as e:
        gpu_quantize(W)
    assert e.value.status == 4


def _c1(seed=0, T=64, n_in=512, n_out=512, r=8, alpha=16.0, zero_B=False):
    W = ss.normal_f32(seed, "c1.W", (n_out, n_in), std=0.02)
    x = ss.to_bf16_values(ss.normal_f32(seed, "c1.x", (T, n_in)))
    A = ss.to_bf16_values(ss.normal_f32(seed, "c1.A", (r, n_in), std=0.02))
    B = np.zeros((n_out, r), np.float32) if zero_B else ss.to_bf16_values(
        ss.normal_f32(seed, "c1.B", (n_out, r), std=0.02))
    dy = ss.to_bf16_values(ss.normal_f32(seed, "c1.dy", (T, n_out)))
    return W, x, A, B, dy, r, alpha / r


def run_gpu_lora(W32, x, A, B, dy, r, s, kind="nf4"):
    T, n_in = x.shape
    n_out = W32.shape[0]
    if kind == "nf4":
        codes, absmax = gpu_quantize(W32)
        Wd = L.weight_nf4(codes, absmax, n_out, n_in)
        keep = (codes, absmax)
        deq = onf4.dequant_bf16(*onf4.quantize(W32))
    else:
        deq = onf4.round_to_bf16(W32)
        wb = dev_bf16(deq)
        Wd = L.weight_bf16(wb)
        keep = (wb,)
    xd, Ad, Bd, dyd = dev_bf16(x), dev_bf16(A), dev_bf16(B), dev_bf16(dy)
    ldT = (T + 7) // 8 * 8
    y = torch.empty((T, n_out), dtype=torch.bfloat16, device="cuda")
    u = torch.zeros((r, ldT), dtype=torch.bfloat16, device="cuda")
    L.soup_lora_linear_fwd(Wd, Ad, Bd, r, s, xd, T, y, u)
    dx = torch.empty((T, n_in), dtype=torch.bfloat16, device="cuda")
    dA = torch.empty((r, n_in), dtype=torch.float32, device="cuda")
    dB = torch.empty((n_out, r), dtype=torch.float32, device="cuda")
    ws = torch.empty(L.soup_lora_linear_bwd_workspace(T, r, n_out), dtype=torch.uint8, device="cuda")
    L.soup_lora_linear_bwd(Wd, Ad, Bd, r, s, xd, u, dyd, T, dx, dA, dB, ws)
    torch.cuda.synchronize()
    del keep
    return dict(y=host(y), u=host(u[:, :T]), dx=host(dx), dA=host(dA), dB=host(dB), deq=deq)


@pytest.mark.parametrize("kind", ["nf4", "bf16"])
@pytest.mark.parametrize("T", [64, 200, 1])
def test_lora_linear_matches_oracle(kind, T):
    W, x, A, B, dy, r, s = _c1(T=T)
    g = run_gpu_lora(W, x, A, B, dy, r, s, kind)
    Wd = g["deq"].astype(np.float64)
    y, u = lora_fwd(x, Wd, A, B, s)
    dx, dA, dB = lora_bwd(x, Wd, A, B, s, dy)
    assert_close(g["y"], y, "y")
    assert_close(g["u"], s * u.T, "u_save")
    assert_close(g["dx"], dx, "dx")
    assert_close(g["dA"], dA, "dA")
    assert_close(g["dB"], dB, "dB")


def test_lora_linear_tiles_and_ragged_tail():
    # several 128-row tiles with a ragged last one, r = 16, N spanning 3 tiles
    W, x, A, B, dy, r, s = _c1(seed=3, T=300, n_in=1024, n_out=768, r=16, alpha=32.0)
    g = run_gpu_lora(W, x, A, B, dy, r, s, "nf4")
    Wd = g["deq"].astype(np.float64)
    y, u = lora_fwd(x, Wd, A, B, s)
    dx, dA, dB = lora_bwd(x, Wd, A, B, s, dy)
    for k, ref in (("y", y), ("dx", dx), ("dA", dA), ("dB", dB)):
        assert_close(g[k], ref, k)


# (T, in, out): one-pair-per-M-tile decode (1 M tile of 256), and decode
# shared by groups of 4 (ragged last M tile) and 8 CTA pairs, forward (W)
# and backward (W^T) layouts
@pytest.mark.parametrize("T,n_in,n_out", [(256, 1024, 1024), (1000, 1024, 768), (2048, 2048, 1536)])
def test_fused_nf4_equals_dequant_then_bf16_gemm_bit_exact(T, n_in, n_out):
    W, x, A, B, dy, r, s = _c1(seed=5, T=T, n_in=n_in, n_out=n_out, r=16, alpha=32.0)
    g_nf4 = run_gpu_lora(W, x, A, B, dy, r, s, "nf4")
    # bf16 path on exactly the dequantised weights
    wb = dev_bf16(g_nf4["deq"])
    Wd = L.weight_bf16(wb)
    xd, Ad, Bd, dyd = dev_bf16(x), dev_bf16(A), dev_bf16(B), dev_bf16(dy)
    ldT = (T + 7) // 8 * 8
    y = torch.empty((T, n_out), dtype=torch.bfloat16, device="cuda")
    u = torch.zeros((r, ldT), dtype=torch.bfloat16, device="cuda")
    L.soup_lora_linear_fwd(Wd, Ad, Bd, r, s, xd, T, y, u)
    dx = torch.empty((T, n_in), dtype=torch.bfloat16, device="cuda")
    dA = torch.empty((r, n_in), dtype=torch.float32, device="cuda")
    dB = torch.empty((n_out, r), dtype=torch.float32, device="cuda")
    ws = torch.empty(L.soup_lora_linear_bwd_workspace(T, r, n_out), dtype=torch.uint8, device="cuda")
    L.soup_lora_linear_bwd(Wd, Ad, Bd, r, s, xd, u, dyd, T, dx, dA, dB, ws)
    torch.cuda.synchronize()
    assert np.array_equal(host(y), g_nf4["y"])
    assert np.array_equal(host(dx), g_nf4["dx"])


def test_B_zero_reproduces_frozen_base_exactly():
    W, x, A, B, dy, r, s = _c1(seed=7, T=128, zero_B=True)
    g0 = run_gpu_lora(W, x, A, B, dy, r, s, "nf4")
    # the same projection with a different A: with B = 0 the adapter term is
    # exactly zero, so y cannot change
    A2 = ss.to_bf16_values(ss.normal_f32(9, "c1.A2", A.shape, std=0.5))
    g1 = run_gpu_lora(W, x, A2, B, dy, r, s, "nf4")
    assert np.array_equal(g0["y"], g1["y"])
    Wd = g0["deq"].astype(np.float64)
    assert_close(g0["y"], x @ Wd.T, "y(B=0)")


def test_epilogue_16_byte_fallback_bit_exact():
    """Outputs 16- but not 32-byte aligned take the epilogue's 16-byte stores
    instead of its 32-byte ones: the same bits either way."""
    T, n_in, n_out = 300, 1024, 768
    W, x, A, B, dy, r, s = _c1(seed=11, T=T, n_in=n_in, n_out=n_out, r=16, alpha=32.0)
    g = run_gpu_lora(W, x, A, B, dy, r, s, "nf4")
    codes, absmax = gpu_quantize(W)
    Wd = L.weight_nf4(codes, absmax, n_out, n_in)
    xd, Ad, Bd, dyd = dev_bf16(x), dev_bf16(A), dev_bf16(B), dev_bf16(dy)
    ldT = (T + 7) // 8 * 8
    ybuf = torch.empty(T * n_out + 8, dtype=torch.bfloat16, device="cuda")
    y = ybuf[8:].view(T, n_out)  # 16 bytes past a 512-byte aligned allocation
    assert y.data_ptr() % 32 == 16
    u = torch.zeros((r, ldT), dtype=torch.bfloat16, device="cuda")
    L.soup_lora_linear_fwd(Wd, Ad, Bd, r, s, xd, T, y, u)
    dxbuf = torch.empty(T * n_in + 8, dtype=torch.bfloat16, device="cuda")
    dx = dxbuf[8:].view(T, n_in)
    dA = torch.empty((r, n_in), dtype=torch.float32, device="cuda")
    dB = torch.empty((n_out, r), dtype=torch.float32, device="cuda")
    ws = torch.empty(L.soup_lora_linear_bwd_workspace(T, r, n_out), dtype=torch.uint8, device="cuda")
    L.soup_lora_linear_bwd(Wd, Ad, Bd, r, s, xd, u, dyd, T, dx, dA, dB, ws)
    torch.cuda.synchronize()
    assert np.array_equal(host(y), g["y"])
    assert np.array_equal(host(dx), g["dx"])
    assert np.array_equal(host(dA), g["dA"])
    assert np.array_equal(host(dB), g["dB"])

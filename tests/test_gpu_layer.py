"""GPU parity of one decoder layer (forward and recompute-backward) against
the CPU oracle, through the C ABI: h_out, dh_in and every LoRA gradient within
relative Frobenius <= 5e-3 and max |diff| <= 1e-2 max |ref|.  Also: adapters
off == B = 0 == frozen base, bit for bit; the backward is deterministic."""
import numpy as np
import pytest
import torch

import soup_synth as ss
from oracle.layer import layer_bwd, layer_fwd
from tests.gpu_util import assert_close, dev_bf16, dev_f32, host
from tests.layer_fixture import DevLayer

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


SMALL = ss.tiny_layer_shape(hidden=512, n_q=4, n_kv=2, head_dim=128, inter=1024, rank=16, alpha=32.0)


def run_layer(dl, h, dh, B, S, on=True):
    T = B * S
    ws = torch.empty(L.soup_decoder_layer_workspace(dl.cfg, B, S), dtype=torch.uint8, device="cuda")
    hd = dev_bf16(h.reshape(T, -1))
    out = torch.empty_like(hd)
    L.soup_decoder_layer_fwd(dl.W, dl.lora, dl.cfg, hd, B, S, out, on, ws)
    dho = dev_f32(dh.reshape(T, -1))
    dhi = torch.empty_like(dho)
    L.soup_decoder_layer_bwd(dl.W, dl.lora, dl.cfg, hd, dho, B, S, dhi, dl.grads, on, ws)
    torch.cuda.synchronize()
    return host(out).reshape(h.shape), host(dhi).reshape(h.shape)


def inputs(shape, B, S, seed=1):
    h = ss.to_bf16_values(ss.normal_f32(seed, "layer.h", (B, S, shape.hidden)))
    dh = ss.to_bf16_values(ss.normal_f32(seed, "layer.dh", (B, S, shape.hidden)))
    return h, dh


@pytest.mark.parametrize("kind", ["nf4", "bf16"])
@pytest.mark.parametrize("B,S", [(2, 100), (1, 256)])
def test_layer_matches_oracle(kind, B, S):
    shape = SMALL
    dl = DevLayer(L, shape, seed=0, kind=kind)
    h, dh = inputs(shape, B, S)
    out, dhi = run_layer(dl, h, dh, B, S)
    ref, cache = layer_fwd(h, dl.Wd, dl.lora_np, shape)
    dref, gref = layer_bwd(cache, dl.Wd, dl.lora_np, shape, dh)
    assert_close(out, ref, "h_out")
    assert_close(dhi, dref, "dh_in")
    got = dl.split_grads()
    for p in ss.PROJ_NAMES:
        assert_close(got[p][0], gref[p][0], f"dA_{p}")
        assert_close(got[p][1], gref[p][1], f"dB_{p}")


def test_layer_adapters_off_equals_B_zero_bit_exact():
    shape = SMALL
    B, S = 1, 192
    h, dh = inputs(shape, B, S, seed=2)
    on = DevLayer(L, shape, seed=3, kind="nf4")
    zero = DevLayer(L, shape, seed=3, kind="nf4", zero_B=True)
    out_off, _ = run_layer(on, h, dh, B, S, on=False)
    out_zero, _ = run_layer(zero, h, dh, B, S, on=True)
    out_on, _ = run_layer(on, h, dh, B, S, on=True)
    assert np.array_equal(out_off, out_zero)
    assert not np.array_equal(out_on, out_off)
    ref, _ = layer_fwd(h, on.Wd, on.lora_np, shape, adapters_on=False)
    assert_close(out_off, ref, "h_out(adapters off)")


def test_layer_backward_is_deterministic():
    shape = SMALL
    B, S = 2, 130
    dl = DevLayer(L, shape, seed=4, kind="nf4")
    h, dh = inputs(shape, B, S, seed=5)
    o1, d1 = run_layer(dl, h, dh, B, S)
    g1 = {k: v.clone() for k, v in dl.grads_t.items()}
    o2, d2 = run_layer(dl, h, dh, B, S)
    assert np.array_equal(o1, o2) and np.array_equal(d1, d2)
    for k in g1:
        assert torch.equal(g1[k], dl.grads_t[k]), k


@pytest.mark.parametrize("kind", ["nf4", "bf16"])
def test_kept_qkv_backward_is_bit_identical(kind):
    """fwd_keep + bwd_kept (q|k|v kept from the forward pass, the backward's
    q|k|v GEMM skipped) gives exactly the gradients and dh_in of fwd + the
    recompute backward, and a forward output within the oracle tolerance."""
    shape = SMALL
    B, S = 2, 130
    T = B * S
    dl = DevLayer(L, shape, seed=6, kind=kind)
    h, dh = inputs(shape, B, S, seed=7)
    o1, d1 = run_layer(dl, h, dh, B, S)
    g1 = {k: v.clone() for k, v in dl.grads_t.items()}
    ws = torch.empty(L.soup_decoder_layer_workspace(dl.cfg, B, S), dtype=torch.uint8, device="cuda")
    keep = torch.empty(L.soup_decoder_layer_keep_bytes(dl.cfg, B, S) // 2, dtype=torch.float16, device="cuda")
    hd = dev_bf16(h.reshape(T, -1))
    out = torch.empty_like(hd)
    L.soup_decoder_layer_fwd_keep(dl.W, dl.lora, dl.cfg, hd, B, S, out, 1, keep, ws)
    dho = dev_f32(dh.reshape(T, -1))
    dhi = torch.empty_like(dho)
    for v in dl.grads_t.values():
        v.zero_()
    L.soup_decoder_layer_bwd_kept(dl.W, dl.lora, dl.cfg, hd, dho, B, S, dhi, dl.grads, 1, keep, ws)
    torch.cuda.synchronize()
    assert np.array_equal(host(dhi).reshape(h.shape), d1)
    for k in g1:
        assert torch.equal(g1[k], dl.grads_t[k]), k
    ref, _ = layer_fwd(h, dl.Wd, dl.lora_np, shape)
    assert_close(host(out).reshape(h.shape), ref, "h_out (q|k|v from the hi + lo input)")
    assert_close(host(out).reshape(h.shape), o1, "h_out vs plain forward", rel=5e-3, maxrel=1e-2)


@pytest.mark.parametrize("h_scale,norm_scale,dh_scale", [
    (32.0, 1.0, 1.0),          # large residual stream (power of two: still bf16-exact)
    (1.0, 4.0, 1.0),           # large normalised activations: q/k/v and g/u (fp16 inside the layer) x4
    (1.0, 1.0, 2.0 ** -14),    # tiny upstream gradient: dO would underflow fp16 without its scale
    (1.0, 1.0, 2.0 ** 10),     # large upstream gradient
])
def test_layer_holds_range(h_scale, norm_scale, dh_scale):
    """Scaled hidden states, RMSNorm weights and upstream gradients (the
    magnitudes real checkpoints produce, which the N(0, 1) inputs of the
    other tests do not reach): the same oracle tolerances hold, so the fp16
    q/k/v, g/u and scaled-dO paths keep their range."""
    shape = SMALL
    B, S = 2, 100
    dl = DevLayer(L, shape, seed=8, kind="nf4")
    if norm_scale != 1.0:
        dl.norm1.mul_(norm_scale)  # powers of two: exact in bf16
        dl.norm2.mul_(norm_scale)
        dl.Wd["norm1"] = dl.Wd["norm1"] * norm_scale
        dl.Wd["norm2"] = dl.Wd["norm2"] * norm_scale
    h, dh = inputs(shape, B, S, seed=9)
    h, dh = h * h_scale, dh * dh_scale
    out, dhi = run_layer(dl, h, dh, B, S)
    ref, cache = layer_fwd(h, dl.Wd, dl.lora_np, shape)
    dref, gref = layer_bwd(cache, dl.Wd, dl.lora_np, shape, dh)
    tag = f"x{h_scale}/{norm_scale}/{dh_scale}"
    assert_close(out, ref, f"h_out {tag}")
    assert_close(dhi, dref, f"dh_in {tag}")
    got = dl.split_grads()
    for p in ss.PROJ_NAMES:
        assert_close(got[p][0], gref[p][0], f"dA_{p} {tag}")
        assert_close(got[p][1], gref[p][1], f"dB_{p} {tag}")


@pytest.mark.parametrize("kind", ["nf4", "bf16"])
def test_saved_layer_backward_is_bit_identical_to_kept(kind):
    """fwd_save + bwd_saved (every intermediate kept, no forward recompute in
    the backward) gives the bits of fwd_keep + bwd_kept (q|k|v kept, the rest
    recomputed): h_out, dh_in and every LoRA gradient."""
    shape = SMALL
    B, S = 2, 130
    T = B * S
    dl = DevLayer(L, shape, seed=6, kind=kind)
    h, dh = inputs(shape, B, S, seed=7)
    ws = torch.empty(L.soup_decoder_layer_workspace(dl.cfg, B, S), dtype=torch.uint8, device="cuda")
    hd = dev_bf16(h.reshape(T, -1))
    dho = dev_f32(dh.reshape(T, -1))
    keep = torch.empty(L.soup_decoder_layer_keep_bytes(dl.cfg, B, S) // 2, dtype=torch.float16, device="cuda")
    out_k = torch.empty_like(hd)
    dhi_k = torch.empty_like(dho)
    L.soup_decoder_layer_fwd_keep(dl.W, dl.lora, dl.cfg, hd, B, S, out_k, 1, keep, ws)
    L.soup_decoder_layer_bwd_kept(dl.W, dl.lora, dl.cfg, hd, dho, B, S, dhi_k, dl.grads, 1, keep, ws)
    torch.cuda.synchronize()
    g_k = {k: v.clone() for k, v in dl.grads_t.items()}
    for v in dl.grads_t.values():
        v.zero_()
    saved = torch.empty(L.soup_decoder_layer_saved_bytes(dl.cfg, B, S), dtype=torch.uint8, device="cuda")
    assert saved.numel() < ws.numel()
    out_s = torch.empty_like(hd)
    dhi_s = torch.empty_like(dho)
    L.soup_decoder_layer_fwd_save(dl.W, dl.lora, dl.cfg, hd, B, S, out_s, 1, saved, ws)
    ws.fill_(0xFF)  # nothing the backward reads may come from the workspace of the forward call
    L.soup_decoder_layer_bwd_saved(dl.W, dl.lora, dl.cfg, hd, dho, B, S, dhi_s, dl.grads, 1, saved, ws)
    torch.cuda.synchronize()
    assert torch.equal(out_s, out_k)
    assert torch.equal(dhi_s, dhi_k)
    for k in g_k:
        assert torch.equal(g_k[k], dl.grads_t[k]), k

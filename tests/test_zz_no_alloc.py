"""The allocation-free LoRA backward (soup_lora_linear_bwd_noalloc), for
callers that cannot allocate device memory when they run the backward (for
example when another allocator's pool owns all device memory, or on a
latency-critical path where cudaMalloc is not allowed).

Through the C ABI it must give what soup_lora_linear_bwd gives with a
caller-provided workspace, within the tolerance the other GPU tests use, on
two calls in a row (the static scratch keeps the previous call's contents),
and it must refuse sizes beyond its static maximum with a clear error.
This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import soup_synth as ss
from tests.gpu_util import assert_close, dev_bf16, dev_f32, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from layer_streamed_qlora_b200 import _lib as lib
    lib.lib()
    return lib


def _problem(L, T=300, n_in=1024, n_out=768, r=16, seed=11):
    W = ss.normal_f32(seed, "na.W", (n_out, n_in), std=0.02)
    x = ss.to_bf16_values(ss.normal_f32(seed, "na.x", (T, n_in)))
    A = ss.to_bf16_values(ss.normal_f32(seed, "na.A", (r, n_in), std=0.02))
    B = ss.to_bf16_values(ss.normal_f32(seed, "na.B", (n_out, r), std=0.02))
    dy = ss.to_bf16_values(ss.normal_f32(seed, "na.dy", (T, n_out)))
    codes = torch.empty((n_out, n_in // 2), dtype=torch.uint8, device="cuda")
    absmax = torch.empty((n_out, n_in // 64), dtype=torch.float32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.soup_nf4_quantize(dev_f32(W), codes, absmax, flag)
    t = dict(codes=codes, absmax=absmax, x=dev_bf16(x), A=dev_bf16(A), B=dev_bf16(B), dy=dev_bf16(dy))
    t["W"] = L.weight_nf4(codes, absmax, n_out, n_in)
    ldT = (T + 7) // 8 * 8
    t["u"] = torch.zeros((r, ldT), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((T, n_out), dtype=torch.bfloat16, device="cuda")
    L.soup_lora_linear_fwd(t["W"], t["A"], t["B"], r, 2.0, t["x"], T, y, t["u"])
    return t, T, n_in, n_out, r


def _outs(T, n_in, n_out, r):
    return (torch.full((T, n_in), float("nan"), dtype=torch.bfloat16, device="cuda"),
            torch.full((r, n_in), float("nan"), dtype=torch.float32, device="cuda"),
            torch.full((n_out, r), float("nan"), dtype=torch.float32, device="cuda"))


def test_noalloc_matches_workspace_backward_twice(L):
    t, T, n_in, n_out, r = _problem(L)
    dx0, dA0, dB0 = _outs(T, n_in, n_out, r)
    ws = torch.empty(L.soup_lora_linear_bwd_workspace(T, r, n_out), dtype=torch.uint8, device="cuda")
    L.soup_lora_linear_bwd(t["W"], t["A"], t["B"], r, 2.0, t["x"], t["u"], t["dy"], T, dx0, dA0, dB0, ws)
    torch.cuda.synchronize()
    ref = (host(dx0), host(dA0), host(dB0))
    for call in range(2):
        dx, dA, dB = _outs(T, n_in, n_out, r)
        L.soup_lora_linear_bwd_noalloc(t["W"], t["A"], t["B"], r, 2.0, t["x"], t["u"], t["dy"], T, dx, dA, dB)
        torch.cuda.synchronize()
        for name, got, want in zip(("dx", "dA", "dB"), (host(dx), host(dA), host(dB)), ref):
            assert_close(got, want, f"call {call}: {name}")
    assert L.device_error() == 0


def test_noalloc_refuses_sizes_beyond_its_scratch(L):
    cap = L.soup_lora_linear_bwd_noalloc_max_scratch()
    assert cap == 8 << 20
    t, T, n_in, n_out, r = _problem(L, T=64, n_in=128, n_out=64, r=16)
    big_T = cap  # r * T * 2 bytes of g' alone exceeds the maximum
    assert L.soup_lora_linear_bwd_workspace(big_T, r, n_out) > cap
    dx, dA, dB = _outs(T, n_in, n_out, r)
    with pytest.raises(L.SoupError) as e:
        L.soup_lora_linear_bwd_noalloc(t["W"], t["A"], t["B"], r, 2.0, t["x"], t["u"], t["dy"], big_T, dx, dA, dB)
    assert e.value.status == 2
    assert "static maximum" in str(e.value)
    torch.cuda.synchronize()
    assert torch.isnan(dA).all()  # nothing ran


def _free_bytes():
    free, _ = torch.cuda.mem_get_info()
    return free


def test_noalloc_allocates_nothing_and_fills_its_whole_scratch(L):
    """A size whose scratch is exactly the static maximum (r = 16, out = 64,
    a ragged T with round_up8(T) * r * 2 + the B^T part = 8 MiB): the second
    call leaves the device's free memory and torch's allocated bytes
    unchanged, and both calls match the workspace path."""
    cap = L.soup_lora_linear_bwd_noalloc_max_scratch()
    r, n_out, n_in = 16, 64, 128
    T = (cap - 256 * ((r * n_out * 2 + 255) // 256)) // (2 * r) - 5  # ragged: round_up8(T) lands on the limit
    need = L.soup_lora_linear_bwd_workspace(T, r, n_out)
    assert cap - 256 < need <= cap, (T, need, cap)
    t, T, n_in, n_out, r = _problem(L, T=T, n_in=n_in, n_out=n_out, r=r, seed=12)
    dx0, dA0, dB0 = _outs(T, n_in, n_out, r)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    L.soup_lora_linear_bwd(t["W"], t["A"], t["B"], r, 2.0, t["x"], t["u"], t["dy"], T, dx0, dA0, dB0, ws)
    torch.cuda.synchronize()
    ref = (host(dx0), host(dA0), host(dB0))
    del ws, dx0, dA0, dB0
    outs = [_outs(T, n_in, n_out, r) for _ in range(2)]
    for call in range(2):
        dx, dA, dB = outs[call]
        torch.cuda.synchronize()
        free0, alloc0 = _free_bytes(), torch.cuda.memory_allocated()
        L.soup_lora_linear_bwd_noalloc(t["W"], t["A"], t["B"], r, 2.0, t["x"], t["u"], t["dy"], T, dx, dA, dB)
        torch.cuda.synchronize()
        if call == 1:  # the first call may load the library's module (and its static array)
            assert _free_bytes() == free0, "the allocation-free backward changed the device's free memory"
            assert torch.cuda.memory_allocated() == alloc0
        for name, got, want in zip(("dx", "dA", "dB"), (host(dx), host(dA), host(dB)), ref):
            assert_close(got, want, f"near-limit call {call}: {name}")
    assert L.device_error() == 0

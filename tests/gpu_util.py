"""Helpers for the GPU parity tests: moving bf16-exact numpy arrays to the
device and the tolerance checks (relative Frobenius error <= 5e-3 and
max |diff| <= 1e-2 * max |ref|)."""
import numpy as np
import torch

REL_FRO = 5e-3
MAX_REL = 1e-2


def dev_bf16(a):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    b = t.to(torch.bfloat16)
    assert torch.equal(b.float(), t), "input is not bf16-exact"
    return b.cuda()


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_fro(got, ref):
    ref = np.asarray(ref, np.float64)
    d = np.linalg.norm(np.asarray(got, np.float64) - ref)
    n = np.linalg.norm(ref)
    return d / n if n > 0 else d


def assert_close(got, ref, name, rel=REL_FRO, maxrel=MAX_REL):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite output"
    rf = rel_fro(got, ref)
    md = np.max(np.abs(got - ref)) if ref.size else 0.0
    mr = np.max(np.abs(ref)) if ref.size else 0.0
    assert rf <= rel, f"{name}: rel Frobenius {rf:.3e} > {rel}"
    assert md <= maxrel * mr + 1e-30, f"{name}: max|diff| {md:.3e} > {maxrel} * max|ref| ({mr:.3e})"
    return rf, md / mr if mr else 0.0

"""Pins for the NF4 oracle (CPU).  Each check uses a route other than the
oracle's own: exact rational brute force, the codebook's construction from
normal quantiles, a hand-worked block, PyTorch's bf16 conversion, and
algebraic invariants (idempotence, sign symmetry of the extremes)."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
CB = nf4.NF4_CODEBOOK


def test_codebook_invariants():
    assert CB.dtype == np.float32 and CB.shape == (16,)
    assert np.all(np.diff(CB.astype(np.float64)) > 0)
    assert CB[0] == -1.0 and CB[7] == 0.0 and CB[15] == 1.0
    assert np.sum(CB < 0) == 7 and np.sum(CB > 0) == 8


def _norm_ppf_bisect(p: float) -> float:
    """Standard normal quantile by bisection on erfc (independent of scipy)."""
    lo, hi = -10.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if 0.5 * math.erfc(-mid / math.sqrt(2.0)) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def _construct(grid_pos, grid_neg, ppf):
    pos = [ppf(float(p)) for p in grid_pos]
    neg = [-ppf(float(p)) for p in grid_neg]
    v = np.sort(np.array(pos + [0.0] + neg)).astype(np.float32)
    return (v / v.max()).astype(np.float32)


# offset of the outermost quantile: halfway between 1 - 1/(2*15) and 1 - 1/(2*16)
DELTA = 0.5 * ((1 - 1 / 30) + (1 - 1 / 32))


def test_codebook_matches_quantile_construction_fp64_grid():
    """8 positive levels at N(0,1) quantiles of 8 evenly spaced probabilities
    in [delta, 1/2), 7 negative ones from 7 in [delta, 1/2), an exact zero,
    normalised by the largest.  With the grid in fp64 the result agrees to a
    few fp32 ulps (the printed table was made on an fp32 grid)."""
    d = round(DELTA, 7)  # the printed offset, 0.9677083
    v = _construct(np.linspace(d, 0.5, 9)[:-1], np.linspace(d, 0.5, 8)[:-1], _norm_ppf_bisect)
    ulps = np.abs(v.view(np.int32).astype(np.int64) - CB.view(np.int32).astype(np.int64))
    assert ulps.max() <= 16, ulps


def test_codebook_matches_quantile_construction_fp32_grid_exactly():
    """Same construction with the probability grid rounded to fp32 the way a
    float32 linspace rounds it: every entry matches bit for bit."""
    torch = pytest.importorskip("torch")
    from scipy.stats import norm
    d = 0.9677083
    gp = torch.linspace(d, 0.5, 9)[:-1].numpy().astype(np.float64)
    gn = torch.linspace(d, 0.5, 8)[:-1].numpy().astype(np.float64)
    v = _construct(gp, gn, lambda p: float(norm.ppf(p)))
    assert np.array_equal(v.view(np.int32), CB.view(np.int32))


def test_round_to_bf16_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        # exact ties: low 16 bits = 0x8000, both parities of the kept lsb
        (np.array([0x3F808000, 0x3F818000, 0xBF808000, 0x40018000, 0x00008000], np.uint32)).view(np.float32),
        np.array([0.0, -0.0, 1e-40, 3.0e38], np.float32),
    ])
    ours = nf4.round_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def _brute_code(w: float, absmax: float) -> int:
    """Exact rational nearest code, ties to the lower index."""
    if absmax == 0.0:
        return 7
    n = Fraction(float(np.float32(np.float32(w) / np.float32(absmax))))
    best, bi = None, -1
    for i, c in enumerate(CB):
        dist = abs(n - Fraction(float(c)))
        if best is None or dist < best:
            best, bi = dist, i
    return bi


def test_quantize_brute_force_tiny_blocks():
    rng = np.random.default_rng(7)
    W = (rng.standard_normal((6, 128)) * 0.02).astype(np.float32)
    W[2, 64:] = rng.uniform(-1, 1, 64).astype(np.float32)
    codes, absmax = nf4.quantize_codes(W)
    for r in range(W.shape[0]):
        for j in range(W.shape[1]):
            assert codes[r, j] == _brute_code(W[r, j], absmax[r, j // 64]), (r, j)
        for b in range(2):
            assert absmax[r, b] == np.max(np.abs(W[r, 64 * b:64 * (b + 1)]))


def test_quantize_midpoint_ties_go_to_lower_index():
    """Blocks whose absmax is 1 and whose elements sit exactly on an
    fp32-representable midpoint between two codes."""
    mids = []
    for i in range(15):
        m = (Fraction(float(CB[i])) + Fraction(float(CB[i + 1]))) / 2
        f = float(np.float32(float(m)))
        if Fraction(f) == m:
            mids.append((i, f))
    assert len(mids) >= 3          # e.g. between 0 and c8, and c6 and 0
    W = np.zeros((1, 64), np.float32)
    W[0, 0] = 1.0
    for j, (i, f) in enumerate(mids):
        W[0, 1 + j] = f
    codes, _ = nf4.quantize_codes(W)
    for j, (i, f) in enumerate(mids):
        assert codes[0, 1 + j] == i, (i, f)


def test_zero_block_and_extremes():
    W = np.zeros((2, 64), np.float32)
    W[1, 3], W[1, 9] = 0.5, -0.5
    codes, absmax = nf4.quantize_codes(W)
    assert absmax[0, 0] == 0 and np.all(codes[0] == 7)
    assert codes[1, 3] == 15 and codes[1, 9] == 0
    deq = nf4.dequant_bf16(nf4.pack(codes), absmax)
    assert np.all(deq[0] == 0)
    assert deq[1, 3] == 0.5 and deq[1, 9] == -0.5


def test_nonfinite_refused():
    W = np.zeros((1, 64), np.float32)
    W[0, 5] = np.nan
    with pytest.raises(ValueError):
        nf4.quantize(W)
    W[0, 5] = np.inf
    with pytest.raises(ValueError):
        nf4.quantize(W)


def test_worked_block_fixture():
    rows = {}
    with open(os.path.join(GOLDEN, "nf4_worked_block.txt")) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            k, v = line.split(":", 1)
            rows[k.strip()] = v.split()
    w = np.zeros((1, 64), np.float32)
    vals = [float(t) for t in rows["weights"]]
    w[0, :len(vals)] = vals
    packed, absmax = nf4.quantize(w)
    codes = nf4.unpack(packed)[0]
    exp_codes = [int(t) for t in rows["codes"]]
    assert list(codes[:len(exp_codes)]) == exp_codes
    assert np.all(codes[len(exp_codes):] == 7)
    assert absmax[0, 0] == float(rows["absmax"][0])
    assert bytes(packed[0]).hex().upper() == "".join(rows["packed_hex"])


def test_pack_nibble_order():
    codes = np.array([[1, 2, 3, 4] * 16], np.uint8)
    p = nf4.pack(codes)
    assert p.shape == (1, 32) and p[0, 0] == 0x12 and p[0, 1] == 0x34
    assert np.array_equal(nf4.unpack(p), codes)


def test_dequant_is_single_fp32_multiply():
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, (4, 128)).astype(np.uint8)
    absmax = (rng.uniform(0.001, 3, (4, 2))).astype(np.float32)
    got = nf4.dequant_fp32(nf4.pack(codes), absmax)
    for r in range(4):
        for j in range(128):
            # fp64 product of two fp32 values is exact; one rounding to fp32
            exp = np.float32(float(CB[codes[r, j]]) * float(absmax[r, j // 64]))
            assert got[r, j] == exp


def test_quantize_dequant_idempotent_on_codebook_exact_inputs():
    """W = c_k * 2^e with every block holding a +-1 code: quantise, dequantise
    (fp32), quantise again gives the same codes and absmax, and dequant
    reproduces W exactly."""
    rng = np.random.default_rng(11)
    codes = rng.integers(0, 16, (8, 256)).astype(np.uint8)
    codes[:, ::64] = 15
    codes[:, 1::64] = 0
    scale = (2.0 ** rng.integers(-8, 3, (8, 4))).astype(np.float32)
    W = (CB[codes].reshape(8, 4, 64) * scale[:, :, None]).reshape(8, 256).astype(np.float32)
    p1, a1 = nf4.quantize(W)
    assert np.array_equal(nf4.unpack(p1), codes)
    assert np.array_equal(a1, scale)
    W2 = nf4.dequant_fp32(p1, a1)
    assert np.array_equal(W2, W)
    p2, a2 = nf4.quantize(W2)
    assert np.array_equal(p2, p1) and np.array_equal(a2, a1)


def test_symmetry_of_extremes():
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((16, 64)) * 0.02).astype(np.float32)
    codes, _ = nf4.quantize_codes(W)
    am_idx = np.argmax(np.abs(W), axis=1)
    for r in range(16):
        assert codes[r, am_idx[r]] == (15 if W[r, am_idx[r]] > 0 else 0)

"""NF4 block quantisation (oracle; test infrastructure only).

Follows the pages' ``quantization: 4bit`` (NF4) frozen base (Soup pages,
"configuration and training" and the published-numbers table: Llama-3.1-8B
NF4) with the data type defined by QLoRA (Dettmers et al. 2023, section 3,
"4-bit NormalFloat quantization"; the 16 values are the ones listed in that
paper's appendix on the NF4 data type).  The pages do not print the
codebook; the readings below fill what they leave open.

Readings
  * block = 64 consecutive elements along the input dimension of a row;
  * absmax = max |w| over the block, in fp32 (exact);
  * n = w / absmax, an IEEE fp32 correctly-rounded division;
  * code = argmin_i |n - c_i| in exact arithmetic, ties to the LOWER index;
  * an all-zero block has absmax 0 and every code 7 (the exact zero);
  * packing: byte j of a row holds element 2j in bits 7..4 and element 2j+1
    in bits 3..0;
  * dequant value = RNE_bf16( fp32(c_code * absmax) ): one fp32 multiply,
    then round-to-nearest-even to bf16;
  * any non-finite weight is refused.
"""
from __future__ import annotations

import numpy as np

BLOCK = 64

# The NormalFloat-4 codebook of QLoRA (16 fp32 values, ascending).  Pinned in
# tests/test_oracle_nf4.py against its construction from N(0,1) quantiles.
NF4_CODEBOOK = np.array([
    -1.0, -0.6961928009986877, -0.5250730514526367, -0.39491748809814453,
    -0.28444138169288635, -0.18477343022823334, -0.09105003625154495, 0.0,
    0.07958029955625534, 0.16093020141124725, 0.24611230194568634,
    0.33791524171829224, 0.44070982933044434, 0.5626170039176941,
    0.7229568362236023, 1.0], dtype=np.float32)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32
    holding the bf16 values.  NaN/Inf are not expected here."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = (u + 0x7FFF + lsb) >> 16
    return (r.astype(np.uint32) << 16).view(np.float32)


def block_absmax(W: np.ndarray) -> np.ndarray:
    out_f, in_f = W.shape
    return np.abs(W.reshape(out_f, in_f // BLOCK, BLOCK)).max(axis=2).astype(np.float32)


def quantize_codes(W: np.ndarray, chunk_rows: int = 512):
    """W fp32 [out, in] -> (codes uint8 [out, in] unpacked 0..15, absmax f32 [out, in/64])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    if W.ndim != 2 or W.shape[1] % BLOCK != 0:
        raise ValueError("W must be [out, in] with in a multiple of 64")
    if not np.all(np.isfinite(W)):
        raise ValueError("non-finite weight")
    out_f, in_f = W.shape
    nb = in_f // BLOCK
    absmax = block_absmax(W)
    codes = np.empty((out_f, in_f), np.uint8)
    cb = NF4_CODEBOOK.astype(np.float64)
    for r0 in range(0, out_f, chunk_rows):
        r1 = min(out_f, r0 + chunk_rows)
        w = W[r0:r1].reshape(r1 - r0, nb, BLOCK)
        am = absmax[r0:r1][:, :, None]
        safe = np.where(am == 0, np.float32(1), am)
        n = (w / safe).astype(np.float32)               # fp32 correctly rounded
        n = np.where(am == 0, np.float32(0), n)
        d = np.abs(n.astype(np.float64)[..., None] - cb)  # exact distances in fp64
        c = np.argmin(d, axis=-1).astype(np.uint8)        # first minimum = lower index
        codes[r0:r1] = c.reshape(r1 - r0, in_f)
    return codes, absmax


def pack(codes: np.ndarray) -> np.ndarray:
    """unpacked codes [out, in] -> bytes [out, in/2], element 2j in the high nibble."""
    hi = codes[:, 0::2].astype(np.uint8)
    lo = codes[:, 1::2].astype(np.uint8)
    return ((hi << 4) | lo).astype(np.uint8)


def unpack(packed: np.ndarray) -> np.ndarray:
    out_f, half = packed.shape
    c = np.empty((out_f, half * 2), np.uint8)
    c[:, 0::2] = packed >> 4
    c[:, 1::2] = packed & 0xF
    return c


def quantize(W: np.ndarray):
    """W fp32 [out, in] -> (packed codes uint8 [out, in/2], absmax f32 [out, in/64])."""
    codes, absmax = quantize_codes(W)
    return pack(codes), absmax


def dequant_fp32(packed: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    """fp32 dequantised weights: c_code * absmax as one fp32 multiply."""
    codes = unpack(packed)
    out_f, in_f = codes.shape
    c = NF4_CODEBOOK[codes].reshape(out_f, in_f // BLOCK, BLOCK)
    v = (c * absmax[:, :, None].astype(np.float32)).astype(np.float32)
    return v.reshape(out_f, in_f)


def dequant_bf16(packed: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    """bf16 dequantised weights (float32 array holding bf16 values)."""
    return round_to_bf16(dequant_fp32(packed, absmax))

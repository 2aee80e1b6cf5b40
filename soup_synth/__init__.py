"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

This module only draws random numbers and lays them out; it holds none of
the arithmetic of layer-streamed LoRA (no quantisation, no matmul, no
normalisation).  Both sides of every parity test receive exactly the arrays
produced here.

Conventions
-----------
* Every tensor gets its own generator, keyed by ``(seed, name)`` so that adding
  a tensor never shifts the draws of another one.
* Floating-point tensors are drawn as float32 from ``numpy``'s PCG64.
* "bf16 inputs" are float32 draws converted to bfloat16 by PyTorch's own
  round-to-nearest-even conversion (a library routine, not ours); they are
  returned as float32 arrays whose values are exactly representable in bf16,
  plus helpers to view them as uint16 bit patterns.

Workload recipes (shapes and distributions) follow the configurations of the
layer-streaming LoRA workloads: NF4 weights from N(0, 0.02), activations
N(0, 1), RMSNorm weights 1 + 0.02 N(0, 1), LoRA A and B from N(0, 0.02),
token ids uniform over the vocabulary.
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "rng_for", "normal_f32", "to_bf16_values", "bf16_bits", "from_bf16_bits",
    "LayerShape", "LLAMA8B_LAYER", "QWEN3B_LAYER", "tiny_layer_shape",
    "layer_weights_f32", "lora_params", "uniform_ids", "PROJ_NAMES",
]

PROJ_NAMES = ("q", "k", "v", "o", "gate", "up", "down")


def rng_for(seed: int, name: str) -> np.random.Generator:
    """Independent PCG64 stream for tensor ``name`` under ``seed``."""
    return np.random.default_rng([int(seed), zlib.crc32(name.encode())])


def normal_f32(seed: int, name: str, shape, std: float = 1.0, mean: float = 0.0) -> np.ndarray:
    g = rng_for(seed, name)
    a = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    if mean != 0.0:
        a += np.float32(mean)
    return a


def to_bf16_values(a: np.ndarray) -> np.ndarray:
    """float32 array -> float32 array of the nearest bf16 values (torch's RNE)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def bf16_bits(a_bf16_values: np.ndarray) -> np.ndarray:
    """float32 array holding bf16-exact values -> uint16 bit patterns."""
    u = np.ascontiguousarray(a_bf16_values, dtype=np.float32).view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("array holds values that are not bf16-exact")
    return (u >> 16).astype(np.uint16)


def from_bf16_bits(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class LayerShape:
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    intermediate: int
    rank: int
    alpha: float
    eps: float = 1e-5
    theta: float = 5e5
    vocab: int = 0
    n_layers: int = 1

    @property
    def scale(self) -> float:
        return self.alpha / self.rank

    def proj_shape(self, p: str):
        """[out, in] of projection ``p``."""
        H, I = self.hidden, self.intermediate
        q_out = self.n_q_heads * self.head_dim
        kv_out = self.n_kv_heads * self.head_dim
        return {
            "q": (q_out, H), "k": (kv_out, H), "v": (kv_out, H), "o": (H, q_out),
            "gate": (I, H), "up": (I, H), "down": (H, I),
        }[p]


# One Llama-3.1-8B-shaped decoder layer (hidden 4096, 32 q / 8 kv heads of 128,
# SwiGLU 14336, LoRA r=16 alpha=32 on all seven projections).
LLAMA8B_LAYER = LayerShape(hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128,
                           intermediate=14336, rank=16, alpha=32.0, eps=1e-5,
                           theta=5e5, vocab=128256, n_layers=32)

# Qwen2.5-3B-shaped stack (hidden 2048, 16 q / 2 kv heads of 128, SwiGLU 11008),
# un-quantised bf16 base, tied embeddings.  No eps/theta is given for it; the
# Llama values are reused.
QWEN3B_LAYER = LayerShape(hidden=2048, n_q_heads=16, n_kv_heads=2, head_dim=128,
                          intermediate=11008, rank=16, alpha=32.0, eps=1e-5,
                          theta=5e5, vocab=151936, n_layers=36)


def tiny_layer_shape(hidden=64, n_q=4, n_kv=2, head_dim=16, inter=128, rank=2, alpha=4.0,
                     vocab=0, n_layers=1) -> LayerShape:
    return LayerShape(hidden=hidden, n_q_heads=n_q, n_kv_heads=n_kv, head_dim=head_dim,
                      intermediate=inter, rank=rank, alpha=alpha, vocab=vocab, n_layers=n_layers)


def layer_weights_f32(shape: LayerShape, seed: int, layer: int = 0, w_std: float = 0.02):
    """fp32 base weights of one decoder layer: dict proj -> [out, in], plus the
    two RMSNorm weight vectors (``norm1``, ``norm2``) drawn as 1 + 0.02 N(0,1)."""
    out = {}
    for p in PROJ_NAMES:
        out[p] = normal_f32(seed, f"L{layer}.W.{p}", shape.proj_shape(p), std=w_std)
    out["norm1"] = to_bf16_values(normal_f32(seed, f"L{layer}.norm1", (shape.hidden,), std=0.02, mean=1.0))
    out["norm2"] = to_bf16_values(normal_f32(seed, f"L{layer}.norm2", (shape.hidden,), std=0.02, mean=1.0))
    return out


def lora_params(shape: LayerShape, seed: int, layer: int = 0, std: float = 0.02, zero_B: bool = False):
    """bf16-exact LoRA factors: dict proj -> (A [r, in], B [out, r])."""
    out = {}
    for p in PROJ_NAMES:
        o, i = shape.proj_shape(p)
        A = to_bf16_values(normal_f32(seed, f"L{layer}.A.{p}", (shape.rank, i), std=std))
        if zero_B:
            B = np.zeros((o, shape.rank), np.float32)
        else:
            B = to_bf16_values(normal_f32(seed, f"L{layer}.B.{p}", (o, shape.rank), std=std))
        out[p] = (A, B)
    return out


def uniform_ids(seed: int, name: str, shape, vocab: int) -> np.ndarray:
    g = rng_for(seed, name)
    return g.integers(0, vocab, size=shape, dtype=np.int64).astype(np.int32)


def nf4_stored_blocks(seed: int, name: str, out_f: int, in_f: int, w_std: float = 0.02):
    """Stored NF4 weights drawn directly (no quantisation step), shaped like
    the NF4 codes of N(0, w_std) weights: the two extreme levels (+-1, the
    block's absmax element) with probability 1/128 each, the 14 inner levels
    equally likely (NF4 levels are equiprobable quantiles), two independent
    codes per byte (high nibble first); a per-64-block absmax of the size the
    largest of 64 N(0, w_std) draws has (w_std x U[2.0, 3.2]).  Returns
    (uint8 [out_f, in_f/2], float32 [out_f, in_f/64])."""
    g = rng_for(seed, name)
    p = np.full(16, (1.0 - 2.0 / 128) / 14)
    p[0] = p[15] = 1.0 / 128
    codes = g.choice(16, size=(out_f, in_f), p=p).astype(np.uint8)
    packed = (codes[:, 0::2] << 4) | codes[:, 1::2]
    absmax = (w_std * (2.0 + 1.2 * g.random((out_f, in_f // 64)))).astype(np.float32)
    return packed.astype(np.uint8), absmax

"""Seeded synthetic inputs for Gated MLA, shared by the CUDA path and the oracle.

This module holds no arithmetic of the method itself: it only draws random
numbers and quantises them to bfloat16 bit patterns.  Both the CUDA path
(through the C-ABI) and the float64 oracle consume the very same bytes.

Recipe:

* a workload has one integer seed; its k-th tensor is cut into blocks of
  ``BLOCK`` elements (row-major order) and block j is drawn from
  ``Generator(PCG64(SeedSequence(seed, spawn_key=(k, j))))`` with
  ``standard_normal(dtype=float32)``, so the bytes do not depend on how many
  threads draw them;
* each value is multiplied by the tensor's standard deviation in float32 and
  rounded to bfloat16 with round-to-nearest-even;
* hidden states X, explicit Q/K/V/G and the latent cache are N(0, 1);
* a weight with ``fan_in`` inputs is N(0, 1/fan_in) -- W_q, W_c, W_g, W_o have
  fan_in = d_model, W_k and W_v have fan_in = d_c -- which keeps the scaled
  scores near unit variance (foundations tutorial "Le Transformer et
  l'attention", the question on dividing by sqrt(d_k));
* tensor order inside a layer workload: X, W_q, W_c, W_k, W_v, W_g, W_o, then
  the cache.

Weights use the nn.Linear orientation [out_features, in_features], read off the
"X W^T" products of the "Gated MLA" problem page.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

__all__ = [
    "BLOCK",
    "SEEDS",
    "Draw",
    "bf16_bits_from_f32",
    "bf16_bits_from_f64",
    "f64_from_bf16_bits",
    "f32_from_bf16_bits",
    "layer_weights",
    "prefill_qkv",
    "decode_plain_qkv",
]

BLOCK = 1 << 22  # elements per independently seeded block

# Seed per workload: the tiny fp32 forward uses 0; the four B200 workloads use 2..5.
SEEDS = {"tiny": 0, "decode_plain": 2, "prefill_attn": 3, "layer_prefill": 4, "latent_decode": 5}


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return uint16 bits.
    Inputs are finite (no NaN handling needed for synthetic data)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    u = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_bits_from_f64(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (nearest, ties to even) directly, with no
    intermediate float32 rounding; return uint16 bits.

    ``frexp`` gives x = m * 2**e with 0.5 <= |m| < 1, so m * 2**8 lies in
    [128, 256) and ``rint`` (half to even) picks the nearest 8-bit significand;
    the result is exact in float32, whose top 16 bits are the pattern.  Meant
    for values in bfloat16's normal range; zero maps to zero."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    return (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def f32_from_bf16_bits(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns exactly to float32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def f64_from_bf16_bits(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns exactly to float64."""
    return f32_from_bf16_bits(bits).astype(np.float64)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


class Draw:
    """Sequential tensor source for one workload seed (see the module recipe)."""

    def __init__(self, seed: int):
        self.seed = int(seed)
        self.k = 0

    def _block(self, k: int, j: int, n: int, std: float, out: np.ndarray, bf16: bool):
        ss = np.random.SeedSequence(self.seed, spawn_key=(k, j))
        g = np.random.Generator(np.random.PCG64(ss))
        v = g.standard_normal(n, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        out[j * BLOCK: j * BLOCK + n] = bf16_bits_from_f32(v) if bf16 else v

    def normal(self, shape, std: float = 1.0, bf16: bool = True) -> np.ndarray:
        """Next tensor: N(0, std^2); bfloat16 bits (uint16) or, with bf16=False, float32."""
        k = self.k
        self.k += 1
        total = int(np.prod(shape))
        flat = np.empty(total, dtype=np.uint16 if bf16 else np.float32)
        nblk = (total + BLOCK - 1) // BLOCK
        jobs = [(k, j, min(BLOCK, total - j * BLOCK), std, flat, bf16) for j in range(nblk)]
        if nblk <= 1:
            for a in jobs:
                self._block(*a)
        else:
            with ThreadPoolExecutor(_threads()) as ex:
                list(ex.map(lambda a: self._block(*a), jobs))
        return flat.reshape(shape)


def layer_weights(draw: Draw, d_model: int, d_c: int, x_shape=None, bf16: bool = True):
    """X (when ``x_shape`` is given) then W_q, W_c, W_k, W_v, W_g, W_o, in that order."""
    out = {}
    if x_shape is not None:
        out["X"] = draw.normal(x_shape, 1.0, bf16)
    s_d = float(1.0 / np.sqrt(d_model))
    s_c = float(1.0 / np.sqrt(d_c))
    out["W_q"] = draw.normal((d_model, d_model), s_d, bf16)
    out["W_c"] = draw.normal((d_c, d_model), s_d, bf16)
    out["W_k"] = draw.normal((d_model, d_c), s_c, bf16)
    out["W_v"] = draw.normal((d_model, d_c), s_c, bf16)
    out["W_g"] = draw.normal((d_model, d_model), s_d, bf16)
    out["W_o"] = draw.normal((d_model, d_model), s_d, bf16)
    return out


def prefill_qkv(seed: int, B: int, Tq: int, H: int, D: int = 128, Tk: int | None = None, gate: bool = False):
    """Explicit Q [B,Tq,H,D], K and V [B,Tk,H,D] and, optionally, gate logits
    G [B,Tq,H*D]: N(0,1) bfloat16 bit patterns."""
    dr = Draw(seed)
    Tk = Tq if Tk is None else Tk
    out = {"Q": dr.normal((B, Tq, H, D)), "K": dr.normal((B, Tk, H, D)), "V": dr.normal((B, Tk, H, D))}
    if gate:
        out["G"] = dr.normal((B, Tq, H * D))
    return out


def decode_plain_qkv(seed: int, B: int, H: int, Tk: int, D: int = 128):
    """Decode-mode tensors in the [B, H, T, D] layout of the "Softmax over keys"
    page: Q [B,H,1,D], K and V [B,H,Tk,D]."""
    dr = Draw(seed)
    return {"Q": dr.normal((B, H, 1, D)), "K": dr.normal((B, H, Tk, D)), "V": dr.normal((B, H, Tk, D))}

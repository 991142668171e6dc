"""Seeded synthetic inputs for Ring Self-Attention (shared by the oracle tests and the GPU path).

This module draws random numbers and rounds them to storage types. It holds none of the
attention arithmetic, so both sides of a parity check can take their inputs from it
without sharing any of the method.

Generator (one stream per seed):

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
  OOPSLA 2014): output t is the finaliser applied to ``seed + (t + 1) * 0x9E3779B97F4A7C15``.
* Two outputs make one pair of uniforms ``u1 = (a >> 11 + 1) / 2**53`` in (0, 1] and
  ``u2 = (b >> 11) / 2**53`` in [0, 1).
* Box and Muller ("A note on the generation of random normal deviates", Ann. Math.
  Statist. 29, 1958) turn the pair into two independent N(0, 1) draws
  ``r cos(2 pi u2)`` and ``r sin(2 pi u2)`` with ``r = sqrt(-2 ln u1)``, in fp64.

Normal number k of the stream comes from pair k // 2 (cosine for even k, sine for odd k).
Tensors are cut from the stream in the order Q, K, V, dO.

Storage rounding is round-to-nearest-even from fp64, straight to the storage type (no
double rounding through fp32 for bf16).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """Outputs ``start .. start+count-1`` of the SplitMix64 stream of ``seed`` (uint64)."""
    t = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + t * _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def normals(seed: int, start: int, count: int) -> np.ndarray:
    """Normals ``start .. start+count-1`` of the seed's stream, fp64."""
    if count <= 0:
        return np.zeros(0, dtype=np.float64)
    p0 = start // 2
    p1 = (start + count - 1) // 2 + 1
    raw = splitmix64(seed, 2 * p0, 2 * (p1 - p0))
    a = raw[0::2]
    b = raw[1::2]
    u1 = ((a >> np.uint64(11)).astype(np.float64) + 1.0) * (1.0 / 9007199254740992.0)
    u2 = (b >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
    r = np.sqrt(-2.0 * np.log(u1))
    pair = np.empty(2 * (p1 - p0), dtype=np.float64)
    pair[0::2] = r * np.cos(2.0 * math.pi * u2)
    pair[1::2] = r * np.sin(2.0 * math.pi * u2)
    off = start - 2 * p0
    return pair[off:off + count]


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 (ties to even); returns the rounded fp64 values.

    bf16 keeps 8 significant bits and the fp32 exponent range. ``frexp`` gives
    x = m * 2**e with 0.5 <= |m| < 1, so m * 2**8 rounded to an integer (numpy's ``rint``
    rounds ties to even, exactly, in fp64) is the 8-bit significand.
    """
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    if np.any((ax != 0) & (ax < 2.0 ** -126)) or np.any(ax >= 2.0 ** 127):
        raise ValueError("value outside the normal bf16 range")
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def bf16_bits(x_rounded: np.ndarray) -> np.ndarray:
    """Bit patterns (uint16) of fp64 values that are exactly representable in bf16."""
    f = np.asarray(x_rounded, dtype=np.float64).astype(np.float32)
    if not np.array_equal(f.astype(np.float64), x_rounded):
        raise ValueError("values are not bf16-exact")
    u = f.view(np.uint32)
    if np.any(u & np.uint32(0xFFFF)):
        raise ValueError("values are not bf16-exact")
    return (u >> np.uint32(16)).astype(np.uint16)


def round_to_f32(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest fp32 (ties to even); returns the rounded fp64 values."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


@dataclasses.dataclass
class RSAInputs:
    """Q, K, V, dO of shape [B, H, L, d], as the exact values of the storage dtype (fp64)
    and as storage bits (uint16 for bf16, float32 for fp32)."""

    B: int
    H: int
    L: int
    d: int
    dtype: str
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    do: np.ndarray

    def storage(self, name: str) -> np.ndarray:
        x = getattr(self, name)
        if self.dtype == "bf16":
            return bf16_bits(x)
        return x.astype(np.float32)

    def torch(self, name: str, device=None):
        """The tensor in its storage dtype as a torch tensor (host unless ``device`` given)."""
        import torch

        s = self.storage(name)
        if self.dtype == "bf16":
            t = torch.from_numpy(s.view(np.int16).copy()).view(torch.bfloat16)
        else:
            t = torch.from_numpy(s.copy())
        return t if device is None else t.to(device)


def make_inputs(B: int, H: int, L: int, d: int, *, seed: int, dtype: str = "bf16",
                qkv_scale: float | None = None, do_scale: float = 1.0,
                q_extra_scale: float = 1.0) -> RSAInputs:
    """Draw Q, K, V ~ N(0,1) * qkv_scale and dO ~ N(0,1) * do_scale from one stream.

    ``qkv_scale`` defaults to 1/sqrt(d) for bf16 (the transformer-shaped workloads) and 1 for
    fp32. ``q_extra_scale`` multiplies Q only (sharp-attention cases). Values are rounded to
    the storage dtype (RNE) and returned as exact fp64 copies of the stored values.
    """
    if dtype not in ("bf16", "f32"):
        raise ValueError("dtype must be 'bf16' or 'f32'")
    n = B * H * L * d
    if qkv_scale is None:
        qkv_scale = 1.0 / math.sqrt(d) if dtype == "bf16" else 1.0
    z = normals(seed, 0, 4 * n)
    shape = (B, H, L, d)
    rnd = round_to_bf16 if dtype == "bf16" else round_to_f32
    q = rnd(z[0:n].reshape(shape) * (qkv_scale * q_extra_scale))
    k = rnd(z[n:2 * n].reshape(shape) * qkv_scale)
    v = rnd(z[2 * n:3 * n].reshape(shape) * qkv_scale)
    do = rnd(z[3 * n:4 * n].reshape(shape) * do_scale)
    return RSAInputs(B, H, L, d, dtype, q, k, v, do)

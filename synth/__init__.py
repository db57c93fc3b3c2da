"""Seeded, counter-based synthetic inputs for the CSA2 decode path.

This module is the one piece shared by the CUDA path's harness and by the CPU
oracle.  It defines the *inputs* (bf16 activations, fp32 index weights,
planted positions) and holds none of the method's arithmetic: no
quantisation, no scoring, no selection, no attention.

Generator definition
--------------------
Every element is a pure function of (seed, tensor name, element index), so any
slice of a multi-GB tensor can be regenerated on its own, on the CPU or on a
GPU, with identical bits:

* ``h = fmix32(fmix32(lo32(i) ^ k1) ^ ((hi32(i) + k2) mod 2^32))`` where
  ``fmix32`` is the 32-bit finaliser of MurmurHash3 (Appleby) and ``k1, k2``
  are derived from (seed, name) by the same finaliser.  All arithmetic runs in
  int64 tensors on values below 2^49, so no step relies on integer overflow.
* Normal draws use the top 16 bits of ``h`` to index a 65536-entry table of
  standard-normal quantiles ``ndtri((u + 1/2) / 65536)`` rounded to bf16.  The
  table is computed once on the host; indexing is integer-only, so CPU and GPU
  produce the same bf16 bits.
* Uniform U(0,1) fp32 draws are ``(2*(h >> 9) + 1) * 2^-24`` (exact in fp32).

Element index conventions (so that a workload can be regenerated per request):
``idx = ((b * POS_STRIDE + pos) * width + c)`` for per-position rows and
``idx = (b * Q_STRIDE + row) * width + c`` for per-query tensors.
"""
from __future__ import annotations

import zlib
from functools import lru_cache

import numpy as np
import torch

M32 = 0xFFFFFFFF
POS_STRIDE = 1 << 24          # positions per request in the element index space
Q_STRIDE = 1 << 16            # query rows per request in the element index space

__all__ = [
    "fmix32_int", "fmix32", "tensor_keys", "hash_u32", "normal_table",
    "normal_bf16", "uniform_f32", "POS_STRIDE", "Q_STRIDE",
]


def fmix32_int(x: int) -> int:
    """MurmurHash3 32-bit finaliser on a Python int (host-side key derivation)."""
    x &= M32
    x ^= x >> 16
    x = (x * 0x85EBCA6B) & M32
    x ^= x >> 13
    x = (x * 0xC2B2AE35) & M32
    x ^= x >> 16
    return x


def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2^32 for int64 x in [0, 2^32), without any int64 overflow."""
    lo = c & 0xFFFF
    hi = c >> 16
    return (x * lo + (((x * hi) & 0xFFFF) << 16)) & M32


def fmix32(x: torch.Tensor) -> torch.Tensor:
    """MurmurHash3 32-bit finaliser, elementwise on an int64 tensor of u32 values."""
    x = x ^ (x >> 16)
    x = _mul32(x, 0x85EBCA6B)
    x = x ^ (x >> 13)
    x = _mul32(x, 0xC2B2AE35)
    x = x ^ (x >> 16)
    return x


def tensor_keys(seed: int, name: str) -> tuple[int, int]:
    """Two 32-bit stream keys for one named tensor of one seeded workload."""
    n = zlib.crc32(name.encode("utf-8")) & M32
    k1 = fmix32_int(fmix32_int(seed * 0x9E3779B1 + 0x632BE5AB) ^ n)
    k2 = fmix32_int(k1 ^ 0x5BD1E995 ^ fmix32_int(n + 0x1B873593))
    return k1, k2


def hash_u32(idx: torch.Tensor, keys: tuple[int, int]) -> torch.Tensor:
    """Counter-based 32-bit hash of int64 element indices (any device)."""
    k1, k2 = keys
    lo = idx & M32
    hi = idx >> 32
    h = fmix32(lo ^ k1)
    return fmix32(h ^ ((hi + k2) & M32))


@lru_cache(maxsize=None)
def _normal_table_cpu() -> torch.Tensor:
    from scipy.special import ndtri
    u = (np.arange(65536, dtype=np.float64) + 0.5) / 65536.0
    t = torch.from_numpy(ndtri(u).astype(np.float32))
    return t.to(torch.bfloat16)


_TABLES: dict = {}


def normal_table(device) -> torch.Tensor:
    device = torch.device(device)
    key = str(device)
    if key not in _TABLES:
        _TABLES[key] = _normal_table_cpu().to(device)
    return _TABLES[key]


def normal_bf16(seed: int, name: str, idx: torch.Tensor) -> torch.Tensor:
    """N(0,1) draws (bf16) for the given int64 element indices."""
    h = hash_u32(idx, tensor_keys(seed, name))
    return normal_table(idx.device)[h >> 16]


def uniform_f32(seed: int, name: str, idx: torch.Tensor) -> torch.Tensor:
    """U(0,1) fp32 draws, exact multiples of 2^-24 in (0, 1)."""
    h = hash_u32(idx, tensor_keys(seed, name))
    return ((h >> 9) * 2 + 1).to(torch.float32) * (2.0 ** -24)


def row_indices(b: int, start: int, count: int, width: int, stride: int, device) -> torch.Tensor:
    """Element indices of rows [start, start+count) of request b, each `width` wide."""
    base = (b * stride + start) * width
    return base + torch.arange(count * width, dtype=torch.int64, device=device)


def rows_normal_bf16(seed: int, name: str, b: int, start: int, count: int, width: int,
                     device="cpu", stride: int = POS_STRIDE) -> torch.Tensor:
    idx = row_indices(b, start, count, width, stride, device)
    return normal_bf16(seed, name, idx).view(count, width)


def rows_uniform_f32(seed: int, name: str, b: int, start: int, count: int, width: int,
                     device="cpu", stride: int = Q_STRIDE) -> torch.Tensor:
    idx = row_indices(b, start, count, width, stride, device)
    return uniform_f32(seed, name, idx).view(count, width)


def rope_table(n_pos: int, pairs: int, base: float = 10000.0) -> np.ndarray:
    """A RoPE angle table as the _rope calls take it: fp32 [n_pos][pairs][2] holding
    (cos, sin) of p * base^(-i / pairs).  The pages give no frequencies; this is the
    common geometric choice, used as a synthetic input (the library applies any table)."""
    p = np.arange(n_pos, dtype=np.float64)[:, None]
    inv = base ** (-np.arange(pairs, dtype=np.float64) / pairs)
    ang = p * inv[None, :]
    return np.ascontiguousarray(np.stack([np.cos(ang), np.sin(ang)], -1).astype(np.float32))

"""Seeded synthetic inputs for the dynamic short convolution.

This module is shared by the CUDA path's tests/benchmark and by the fp64
oracle's tests.  It holds no arithmetic of the convolution itself: it only
draws numbers and rounds them to the storage dtype, so that both sides see
bit-identical inputs.

Generator (counter based, so any element can be drawn independently):

* SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): with golden gamma ``G = 0x9E3779B97F4A7C15``
  and the finaliser ``mix64``, the i-th output (i = 0, 1, ...) of the
  generator started at state ``s0`` is ``mix64(s0 + (i + 1) * G)``.
* The stream of one tensor starts at
  ``s0 = mix64((seed << 32) | tensor_id)``.
* Element i of a normal tensor uses outputs 2i and 2i+1 with the
  Box-Muller transform (Box & Muller 1958), cosine branch:
  ``u1 = ((a >> 11) + 1) * 2**-53`` in (0, 1],
  ``u2 = (b >> 11) * 2**-53`` in [0, 1),
  ``n = sqrt(-2 ln u1) * cos(2 pi u2)``.
* The fp64 value ``std * n`` is rounded to fp32 (round to nearest even),
  then, for bf16 tensors, to bf16 (round to nearest even on the fp32 bits).

Storage: fp32 tensors are ``numpy.float32`` arrays, bf16 tensors are
``numpy.uint16`` arrays holding the bf16 bit patterns.
"""

from __future__ import annotations

import math
import os

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

F32 = "f32"
BF16 = "bf16"

# Tensor ids of the stream keys (one stream per tensor role).
TID_X, TID_W, TID_Z, TID_U, TID_DY, TID_WS, TID_STATE, TID_H, TID_V = 1, 2, 3, 4, 5, 6, 7, 8, 9

_CHUNK = 1 << 21


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def mix64_scalar(v: int) -> int:
    """SplitMix64 finaliser on one Python int (mod 2**64)."""
    m = (1 << 64) - 1
    v &= m
    v = ((v ^ (v >> 30)) * 0xBF58476D1CE4E5B9) & m
    v = ((v ^ (v >> 27)) * 0x94D049BB133111EB) & m
    return v ^ (v >> 31)


def stream_key(seed: int, tensor_id: int) -> int:
    return mix64_scalar(((seed & 0xFFFFFFFF) << 32) | (tensor_id & 0xFFFFFFFF))


def splitmix_outputs(key: int, first: int, count: int) -> np.ndarray:
    """Outputs first .. first+count-1 of the SplitMix64 stream at state ``key``."""
    idx = np.arange(first + 1, first + 1 + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        s = np.uint64(key) + idx * GAMMA
        return _mix64(s)


def normals_f64(seed: int, tensor_id: int, n: int, start: int = 0) -> np.ndarray:
    """Standard normals for elements start .. start+n-1 of one tensor, in fp64.

    Chunks are drawn on a thread pool; every element depends only on its
    index, so the result does not depend on the chunking or thread count."""
    key = stream_key(seed, tensor_id)
    out = np.empty(n, dtype=np.float64)

    def fill(lo):
        m = min(_CHUNK, n - lo)
        raw = splitmix_outputs(key, 2 * (start + lo), 2 * m)
        a = raw[0::2]
        b = raw[1::2]
        u1 = ((a >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * (2.0 ** -53)
        u2 = (b >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
        out[lo:lo + m] = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)

    starts = range(0, n, _CHUNK)
    if n <= _CHUNK:
        for lo in starts:
            fill(lo)
    else:
        from concurrent.futures import ThreadPoolExecutor

        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, starts))
    return out


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_f64(arr: np.ndarray, dtype: str) -> np.ndarray:
    """Exact fp64 value of a stored tensor."""
    if dtype == BF16:
        return bf16_bits_to_f32(arr).astype(np.float64)
    return np.asarray(arr, dtype=np.float32).astype(np.float64)


def make_tensor(seed: int, tensor_id: int, shape, std: float, dtype: str) -> np.ndarray:
    """A seeded N(0, std**2) tensor of ``shape`` in storage form for ``dtype``."""
    n = int(np.prod(shape)) if len(shape) else 1
    vals = (normals_f64(seed, tensor_id, n) * std).astype(np.float32)
    if dtype == BF16:
        return f32_to_bf16_bits(vals).reshape(shape)
    if dtype == F32:
        return vals.reshape(shape)
    raise ValueError(f"unknown dtype {dtype!r}")


def to_torch(arr: np.ndarray, dtype: str):
    """View a stored tensor as a torch CPU tensor of the matching dtype (no copy)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(arr))
    if dtype == BF16:
        return t.view(torch.bfloat16)
    return t


def from_torch(t, dtype: str) -> np.ndarray:
    """Storage form of a torch tensor (bf16 -> uint16 bits)."""
    import torch

    t = t.detach().contiguous().cpu()
    if dtype == BF16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.to(torch.float32).numpy()

"""Seeded synthetic inputs shared by the tests, the benchmark and the CPU oracle.

This module holds no arithmetic of the attention block: it draws numbers and
stores them in the element formats the library consumes. Both the CUDA path
and the oracle read the same bits, so a bf16 input is rounded once, here, by
round-to-nearest-even, and the oracle upcasts those exact bits.

Recipe: ``numpy.random.default_rng(seed)``; q, k and v are drawn in that order
from one stream with ``standard_normal(dtype=float32)`` times ``std``, in the
full-sequence BSHD shape ``[batch, prefix + tokens, heads, head_dim]`` (k and v
with the workload's kv head count under grouped-query attention).
Bit-pattern inputs for layout tests are uniform random 16- or 32-bit words.
"""

from __future__ import annotations

import numpy as np

from .workloads import Workload


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return uint16 bits.

    Inputs are finite normal draws; NaN is not expected here.
    """
    bits = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((bits >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((bits + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact float32 value of bfloat16 bit patterns."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def storage_to_f64(storage: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of stored elements (bf16 bits or float32)."""
    if dtype == "bf16":
        return bf16_bits_to_f32(storage).astype(np.float64)
    if dtype == "fp32":
        return np.asarray(storage, dtype=np.float64)
    raise ValueError(f"unknown dtype {dtype}")


def full_shape(w: Workload) -> tuple[int, int, int, int]:
    return (w.batch, w.prefix + w.seq_len, w.heads, w.head_dim)


def make_qkv(w: Workload, seed: int | None = None):
    """Full-sequence q, k, v in storage form (uint16 bf16 bits, or float32)."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    shape = full_shape(w)
    kv_shape = shape[:2] + (w.heads_kv,) + shape[3:]
    out = []
    for i in range(3):
        x = rng.standard_normal(size=shape if i == 0 else kv_shape, dtype=np.float32)
        if w.std != 1.0:
            x *= np.float32(w.std)
        out.append(f32_to_bf16_bits(x) if w.dtype == "bf16" else x)
    return tuple(out)


def make_bits(shape, itemsize: int, seed: int) -> np.ndarray:
    """Uniform random bit patterns (NaN payloads, -0 and Inf included by chance
    and by the fixed values planted at the front)."""
    rng = np.random.default_rng(seed)
    dt = {2: np.uint16, 4: np.uint32}[itemsize]
    x = rng.integers(0, np.iinfo(dt).max, size=shape, dtype=dt, endpoint=True)
    flat = x.reshape(-1)
    planted = {2: [0x8000, 0x7F80, 0xFF80, 0x7FC1, 0xFFFF, 0x0001],
               4: [0x80000000, 0x7F800000, 0xFF800000, 0x7FC00001, 0xFFFFFFFF, 0x00000001]}[itemsize]
    n = min(len(planted), flat.size)
    flat[:n] = np.asarray(planted[:n], dtype=dt)
    return x

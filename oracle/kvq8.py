"""8-bit KV-cache entries for long contexts, numpy.

Test infrastructure only (see the package docstring).

Source: the open-jet Qwen3.8-27B megakernel follow-up post ("Limits"): a 147K-token
context fits on one 24 GB card with the KV cache in fp16 up to about 80K positions and
"q8" above. The post does not define the format; the plainest reading is the common
8-bit block format: the entries of one (head, position) vector are cut into blocks of
32 along the head dimension, each block stores one fp16 scale d and 32 signed codes q,
and the entry reads back as d * q. Here

    d = max |x| / 127           (float32 division)
    q = round(x / d)            (float32 division, nearest, ties to even, in [-127, 127])
    stored scale = fp16(d)      (nearest, ties to even); an all-zero block stores d = 0, q = 0

The codes are integers decided by float arithmetic, so the decision is taken in float32
(the precision of the GPU path's activations) from the float32 value of the entry.
"""
from __future__ import annotations

import numpy as np

__all__ = ["Q8_BLOCK", "quantize_q8", "dequantize_q8", "q8_roundtrip"]

Q8_BLOCK = 32


def quantize_q8(x: np.ndarray):
    """x [..., D] (D a multiple of 32) -> (codes int8 [..., D], scales float16 [..., D / 32])."""
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    if x32.shape[-1] % Q8_BLOCK:
        raise ValueError("the last dimension must be a multiple of 32")
    blocks = x32.reshape(*x32.shape[:-1], x32.shape[-1] // Q8_BLOCK, Q8_BLOCK)
    amax = np.abs(blocks).max(axis=-1)
    d = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(d > 0, d, np.float32(1.0)).astype(np.float32)
    q = np.rint((blocks / safe[..., None]).astype(np.float32))
    q = np.where(d[..., None] > 0, np.clip(q, -127, 127), 0).astype(np.int8)
    return q.reshape(x32.shape), d.astype(np.float16)


def dequantize_q8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """(codes [..., D], scales [..., D / 32]) -> float64 [..., D] = scale * code."""
    c = np.asarray(codes, dtype=np.float64)
    blocks = c.reshape(*c.shape[:-1], c.shape[-1] // Q8_BLOCK, Q8_BLOCK)
    out = blocks * np.asarray(scales, dtype=np.float64)[..., None]
    return out.reshape(c.shape)


def q8_roundtrip(x: np.ndarray) -> np.ndarray:
    """The value an entry reads back as after 8-bit storage."""
    return dequantize_q8(*quantize_q8(x))

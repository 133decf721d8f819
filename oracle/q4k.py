"""Q4_K-style 4-bit super-block decoding, float64 numpy.

Test infrastructure only (see the package docstring).

The open-jet megakernel follow-up post ("Quantisation support") runs the 27B model
from Q4_K_M files: 256-weight super-blocks with 4-bit codes, 6-bit sub-block
scales and mins and fp16 super-scales. This library uses its own byte layout of
that format (it does not read GGUF files). One super-block is 144 bytes:

  [0:2]   d     fp16 super-scale of the sub-block scales
  [2:4]   dmin  fp16 super-scale of the sub-block mins
  [4:16]  sixteen 6-bit fields as one little-endian bit stream: sc_0..sc_7, m_0..m_7
  [16:144] 4-bit codes; sub-block j (32 weights) uses bytes 16+16j .. 16+16j+15,
           byte t holds weight 32j+t in its low nibble and 32j+t+16 in its high nibble.

Weight i of sub-block j:  w = (d * sc_j) * q_i - (dmin * m_j).
"""
from __future__ import annotations

import numpy as np

__all__ = ["dequant_q4k_block", "dequant_q4k_matrix", "unpack_q4k_fields"]

BLOCK_BYTES = 144
BLOCK = 256


def unpack_q4k_fields(blk: np.ndarray):
    """One 144-byte block -> (d, dmin, sc[8], m[8], q[256]) with plain Python bit work."""
    blk = np.asarray(blk, dtype=np.uint8)
    d = float(blk[0:2].view(np.float16)[0])
    dmin = float(blk[2:4].view(np.float16)[0])
    stream = 0
    for i in range(12):
        stream |= int(blk[4 + i]) << (8 * i)
    fields = [(stream >> (6 * f)) & 0x3F for f in range(16)]
    sc, m = fields[:8], fields[8:]
    q = np.empty(BLOCK, dtype=np.int64)
    for j in range(8):
        for t in range(16):
            byte = int(blk[16 + 16 * j + t])
            q[32 * j + t] = byte & 0xF
            q[32 * j + t + 16] = byte >> 4
    return d, dmin, sc, m, q


def dequant_q4k_block(blk: np.ndarray) -> np.ndarray:
    d, dmin, sc, m, q = unpack_q4k_fields(blk)
    out = np.empty(BLOCK)
    for j in range(8):
        out[32 * j:32 * j + 32] = (d * sc[j]) * q[32 * j:32 * j + 32] - (dmin * m[j])
    return out


def dequant_q4k_matrix(data: np.ndarray, cols: int) -> np.ndarray:
    """[rows, cols/256*144] bytes -> [rows, cols] float64, vectorised over blocks."""
    data = np.asarray(data, dtype=np.uint8)
    rows = data.shape[0]
    nb = cols // BLOCK
    b = data.reshape(rows, nb, BLOCK_BYTES)
    d = b[:, :, 0:2].copy().view(np.float16)[..., 0].astype(np.float64)
    dmin = b[:, :, 2:4].copy().view(np.float16)[..., 0].astype(np.float64)
    # 96-bit field stream as two integers: bytes 4..11 (low 64 bits) and 12..15
    lo = np.zeros((rows, nb), dtype=np.uint64)
    for i in range(8):
        lo |= b[:, :, 4 + i].astype(np.uint64) << np.uint64(8 * i)
    hi = np.zeros((rows, nb), dtype=np.uint64)
    for i in range(4):
        hi |= b[:, :, 12 + i].astype(np.uint64) << np.uint64(8 * i)
    fields = np.empty((rows, nb, 16), dtype=np.int64)
    for f in range(16):
        bit = 6 * f
        if bit + 6 <= 64:
            v = (lo >> np.uint64(bit)) & np.uint64(0x3F)
        elif bit >= 64:
            v = (hi >> np.uint64(bit - 64)) & np.uint64(0x3F)
        else:
            v = ((lo >> np.uint64(bit)) | (hi << np.uint64(64 - bit))) & np.uint64(0x3F)
        fields[:, :, f] = v.astype(np.int64)
    sc = fields[:, :, :8].astype(np.float64)
    m = fields[:, :, 8:].astype(np.float64)
    codes = b[:, :, 16:].reshape(rows, nb, 8, 16)
    q = np.concatenate([codes & 0xF, codes >> 4], axis=3).astype(np.float64)   # [rows, nb, 8, 32]
    w = (d[..., None] * sc)[..., None] * q - (dmin[..., None] * m)[..., None]
    return w.reshape(rows, cols)

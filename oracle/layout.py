"""Storage layout of NVFP4 tensors, as the oracle reads it.  TEST INFRASTRUCTURE.

The pages fix the format (E2M1 codes, one E4M3 scale per 16 elements) but no
byte layout.  The layout read here is the one the block-scaled tensor-core MMA
consumes; it is stated independently of the CUDA sources and pinned on the GPU
by single-nonzero GEMM probes:

* codes: two per byte, the element with the even column index in the low nibble,
  row-major ``[rows, cols/2]``;
* scales: 128-row x 4-block atoms of 512 bytes.  Inside an atom, row r and block
  j (r < 128, j < 4) sit at byte ``(r % 32) * 16 + (r // 32) * 4 + j``.  Atoms are
  ordered with the block (K) index fastest: atom ``(r // 128) * kb_atoms + j // 4``.
  Rows are padded to a multiple of 128 and blocks to a multiple of 4; padding
  bytes are zero.
"""
from __future__ import annotations

import numpy as np

__all__ = ["pack_nibbles", "unpack_nibbles", "scale_bytes", "swizzle_scales",
           "unswizzle_scales", "scale_offset"]


def pack_nibbles(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    rows, cols = codes.shape
    assert cols % 2 == 0
    lo = codes[:, 0::2] & 0xF
    hi = codes[:, 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_nibbles(packed) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    rows, half = packed.shape
    out = np.empty((rows, half * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def _padded(rows: int, cols: int):
    rows_pad = -(-rows // 128) * 128
    kb = cols // 16
    kb_pad = -(-kb // 4) * 4
    return rows_pad, kb_pad


def scale_bytes(rows: int, cols: int) -> int:
    rows_pad, kb_pad = _padded(rows, cols)
    return rows_pad * kb_pad


def scale_offset(r, j, cols: int):
    """Byte offset of row ``r``, block ``j`` in the swizzled scale buffer."""
    _, kb_pad = _padded(1, cols)
    r = np.asarray(r, dtype=np.int64)
    j = np.asarray(j, dtype=np.int64)
    atom = (r // 128) * (kb_pad // 4) + j // 4
    return atom * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (j % 4)


def swizzle_scales(sf, rows: int, cols: int) -> np.ndarray:
    sf = np.asarray(sf, dtype=np.uint8)
    out = np.zeros(scale_bytes(rows, cols), dtype=np.uint8)
    r, j = np.meshgrid(np.arange(rows), np.arange(cols // 16), indexing="ij")
    out[scale_offset(r, j, cols)] = sf
    return out


def unswizzle_scales(buf, rows: int, cols: int) -> np.ndarray:
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    r, j = np.meshgrid(np.arange(rows), np.arange(cols // 16), indexing="ij")
    return buf[scale_offset(r, j, cols)]

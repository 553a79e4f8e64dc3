"""Shape of the packed sign-matrix buffer (sizes and padding only).

A sign matrix of ``rows x cols`` entries is stored in row tiles of 32 rows and
column quads of 128 columns. Each (tile, quad) block is 32 rows x 4 words of
32 bits, row-major inside the block, so 32 lanes that each own one row of the
tile read 512 contiguous bytes with one 16-byte load apiece. The buffer is
``[tiles][quads][32][4]`` little-endian uint32 words; entries past ``rows`` or
``cols`` are padding and hold bit 0.

This module only sizes buffers and locates padding; it never interprets a bit.
"""

import numpy as np

ROW_TILE = 32
COL_QUAD = 128


def tiles(rows: int) -> int:
    return (rows + ROW_TILE - 1) // ROW_TILE


def quads(cols: int) -> int:
    return (cols + COL_QUAD - 1) // COL_QUAD


def packed_words(rows: int, cols: int) -> int:
    """Number of uint32 words of one packed ``rows x cols`` sign matrix."""
    return tiles(rows) * quads(cols) * ROW_TILE * 4


def zero_padding_bits(words: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Clear the padding entries of a packed buffer of random words in place.

    ``words`` has shape ``[..., packed_words(rows, cols)]``; the leading axes
    (bases) are handled together.
    """
    T, Q = tiles(rows), quads(cols)
    w = words.reshape(words.shape[:-1] + (T, Q, ROW_TILE, 4))
    pad_rows = T * ROW_TILE - rows
    if pad_rows:
        w[..., T - 1, :, ROW_TILE - pad_rows:, :] = 0
    pad_cols = Q * COL_QUAD - cols
    if pad_cols:
        valid = COL_QUAD - pad_cols          # valid columns in the last quad
        for j in range(4):
            lo = 32 * j
            n = min(max(valid - lo, 0), 32)  # valid bits in word j
            mask = np.uint32(0xFFFFFFFF) if n == 32 else np.uint32((1 << n) - 1)
            w[..., Q - 1, :, j] &= mask
    return words

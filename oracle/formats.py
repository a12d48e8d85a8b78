"""The oracle's own reading of the library's packed storage formats.

Test infrastructure: converts between the plain layouts the oracle uses (one
code per byte, row-major ``[rows][K/32]`` scales) and the packed formats the
C-ABI documents, written independently of the CUDA code:

* codes: ``[rows][K/2]`` bytes, element ``2i`` in the low nibble, ``2i+1`` in
  the high nibble;
* scales: rows padded to a multiple of 128 and blocks to a multiple of 4; byte
  of (row m, block b) at ``((m//128)*nbp4 + b//4)*512 + (m%32)*16 + ((m%128)//32)*4 + b%4``
  with ``nbp4 = ceil(nb/4)``.
"""
from __future__ import annotations

import numpy as np


def pack_codes(codes: np.ndarray) -> np.ndarray:
    codes = np.asarray(codes, np.uint8)
    return (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, np.uint8)
    rows, half = packed.shape
    out = np.empty((rows, 2 * half), np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def scale_bytes(rows: int, nb: int) -> int:
    return ((rows + 127) // 128) * ((nb + 3) // 4) * 512


def scale_index(rows: int, nb: int) -> np.ndarray:
    """Index array I with tiled[I[m, b]] = scale of (m, b)."""
    nbp4 = (nb + 3) // 4
    m = np.arange(rows)[:, None]
    b = np.arange(nb)[None, :]
    return ((m // 128) * nbp4 + b // 4) * 512 + (m % 32) * 16 + ((m % 128) // 32) * 4 + b % 4


def untile_scales(tiled: np.ndarray, rows: int, nb: int) -> np.ndarray:
    return np.asarray(tiled, np.uint8).reshape(-1)[scale_index(rows, nb)]


def tile_scales(plain: np.ndarray) -> np.ndarray:
    rows, nb = plain.shape
    out = np.zeros(scale_bytes(rows, nb), np.uint8)
    out[scale_index(rows, nb)] = plain
    return out


def padding_mask(rows: int, nb: int) -> np.ndarray:
    """True at every byte of the tiled buffer that belongs to no (m, b)."""
    mask = np.ones(scale_bytes(rows, nb), bool)
    mask[scale_index(rows, nb).reshape(-1)] = False
    return mask

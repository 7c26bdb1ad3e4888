"""Decoding of the library's NVFP4 storage into the oracle's logical layout (test-side).

Follows the storage definition in include/nvfp4rac.h: two E2M1 codes per byte (element 2j in
the low nibble), scales in 512-byte atoms covering 128 rows x 64 columns, where the scale of
row r (r % 128 = 32 i + j) and 16-column block c sits at byte j*16 + i*4 + (c % 4) of atom
(r // 128, c // 4), atoms ordered row-block major.  In the 16-row slab layout of decode
activations, slab s = r // 16 owns atoms (s, c // 4) and row r uses byte (r % 16)*16 + (c % 4).
"""
import numpy as np


def unpack_codes(codes: np.ndarray, rows: int, rows_padded: int, cols: int) -> np.ndarray:
    b = np.asarray(codes, dtype=np.uint8).reshape(rows_padded, cols // 2)[:rows]
    out = np.empty((rows, cols), dtype=np.uint8)
    out[:, 0::2] = b & 0xF
    out[:, 1::2] = b >> 4
    return out


def sf_index(rows_padded: int, cols: int) -> np.ndarray:
    """Byte offset of every logical scale [rows_padded, cols/16] inside the atom array."""
    r = np.arange(rows_padded)[:, None]
    c = np.arange(cols // 16)[None, :]
    atom = (r // 128) * (cols // 64) + c // 4
    return atom * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (c % 4)


def sf_index_slab16(rows_padded: int, cols: int) -> np.ndarray:
    """sf_index for the 16-row slab layout."""
    r = np.arange(rows_padded)[:, None]
    c = np.arange(cols // 16)[None, :]
    atom = (r // 16) * (cols // 64) + c // 4
    return atom * 512 + (r % 16) * 16 + (c % 4)


def unpack_sf(sf: np.ndarray, rows: int, rows_padded: int, cols: int, slab16: bool = False) -> np.ndarray:
    flat = np.asarray(sf, dtype=np.uint8).reshape(-1)
    idx = sf_index_slab16(rows_padded, cols) if slab16 else sf_index(rows_padded, cols)
    return flat[idx][:rows]


def pack_sf(S: np.ndarray, rows_padded: int) -> np.ndarray:
    """Inverse of unpack_sf for a full [rows_padded, cols/16] matrix."""
    cols = S.shape[1] * 16
    out = np.zeros(rows_padded * cols // 16, dtype=np.uint8)
    out[sf_index(rows_padded, cols)] = S
    return out


def pack_codes(C: np.ndarray) -> np.ndarray:
    C = np.asarray(C, dtype=np.uint8)
    return (C[:, 0::2] | (C[:, 1::2] << 4)).astype(np.uint8).reshape(-1)

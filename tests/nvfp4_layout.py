"""Decoding of the library's NVFP4 storage into the oracle's logical layout (test-side).

Follows the storage definition in include/nvfp4rac.h: two E2M1 codes per byte (element 2j in
the low nibble), scales in 512-byte atoms covering 128 rows x 64 columns, where the scale of
row r (r % 128 = 32 i + j) and 16-column block c sits at byte j*16 + i*4 + (c % 4) of atom
(r // 128, c // 4), atoms ordered row-block major.  In the 16-row slab layout of decode
activations, slab s = r // 16 owns atoms (s, c // 4) and row r uses byte (r % 16)*16 + (c % 4).

Also the expert-grouped row layouts written out on the host (padded segments, scatter lists,
decode slabs): test-side checkers of the device dispatch plan (moe_dispatch_plan) and inputs of
the tests that build a layout by hand.
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


def expert_layout(counts, pad: int = 128):
    """Padded expert segments for a token-sorted pair list.

    counts: pairs per expert.  Returns (offsets_padded [E+1] int64, rows_padded_total, pair_rows [P]) where
    pair_rows maps the i-th (expert, token)-sorted pair to its row in the padded layout.
    """
    import numpy as np

    counts = np.asarray(counts, dtype=np.int64)
    padded = (counts + pad - 1) // pad * pad
    off = np.zeros(counts.size + 1, dtype=np.int64)
    off[1:] = np.cumsum(padded)
    starts = off[:-1]
    pair_rows = np.concatenate([starts[e] + np.arange(c) for e, c in enumerate(counts)]) if counts.sum() else \
        np.zeros(0, np.int64)
    return off, int(off[-1]), pair_rows


def gather_map(pair_token, counts, pad: int = 128):
    """row_gather [rows_padded] (source token of each padded row, -1 for padding) and offsets."""
    import numpy as np

    off, total, pair_rows = expert_layout(counts, pad)
    g = np.full(total, -1, dtype=np.int32)
    g[pair_rows] = np.asarray(pair_token, dtype=np.int32)
    return g, off, pair_rows


def scatter_map(pair_token, pair_rows, T: int, fanout: int):
    """row_scatter [T, fanout]: the padded rows of each token's (token, expert) pairs, -1 padded."""
    import numpy as np

    m = np.full((T, fanout), -1, dtype=np.int32)
    fill = np.zeros(T, dtype=np.int64)
    for t, r in zip(np.asarray(pair_token), np.asarray(pair_rows)):
        m[t, fill[t]] = r
        fill[t] += 1
    return m


def decode_slots(counts, slab: int = 16):
    """16-token slabs for a decode step's (expert, token)-sorted pair list.

    counts: pairs per expert.  Returns (slot_expert [S] int32, slot_count [S] int32, pair_rows [P] int64)
    where expert e's pairs fill ceil(counts[e] / 16) consecutive slabs and pair i lands in row
    16 * slot + j of the slab layout.
    """
    import numpy as np

    counts = np.asarray(counts, dtype=np.int64)
    slot_expert, slot_count, pair_rows = [], [], []
    for e, c in enumerate(counts):
        for k in range(0, int(c), slab):
            n = min(slab, int(c) - k)
            base = len(slot_expert) * slab
            slot_expert.append(e)
            slot_count.append(n)
            pair_rows.extend(range(base, base + n))
    return (np.asarray(slot_expert, dtype=np.int32), np.asarray(slot_count, dtype=np.int32),
            np.asarray(pair_rows, dtype=np.int64))

"""Test-side conversion between plain [rows x k/16] scale arrays and the
library's 128x4 scale-atom layout (see include/nvfp4.h)."""
import numpy as np


def scales_bytes(rows, k):
    if rows <= 0 or k <= 0:
        return 0
    return ((rows + 127) // 128) * 128 * ((k + 63) // 64) * 4


def atom_offsets(rows, k):
    """Byte offset of every (r, b) in the atom layout, shape [rows, k/16]."""
    kb4 = (k + 63) // 64
    r = np.arange(rows, dtype=np.int64)[:, None]
    b = np.arange(k // 16, dtype=np.int64)[None, :]
    return ((r // 128) * kb4 + b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (b % 4)


def atoms_to_plain(buf, rows, k):
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    return buf[atom_offsets(rows, k)]


def plain_to_atoms(plain, rows, k):
    out = np.zeros(max(scales_bytes(rows, k), 16), np.uint8)
    out[atom_offsets(rows, k)] = plain
    return out


def padding_mask(rows, k):
    """True for the bytes of the atom buffer that hold no (r, b) entry."""
    m = np.ones(max(scales_bytes(rows, k), 16), bool)
    m[atom_offsets(rows, k)] = False
    m[scales_bytes(rows, k):] = False
    return m

"""Counter-based random numbers for attention dropout (test infrastructure).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  This is the oracle's own
implementation of Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel
Random Numbers: As Easy as 1, 2, 3", SC 2011), written from that published
definition; the CUDA library implements the same generator independently.

Philox4x32-10: a 128-bit counter (c0, c1, c2, c3) and a 64-bit key (k0, k1)
go through 10 rounds.  One round multiplies c0 and c2 by the constants
M0 = 0xD2511F53 and M1 = 0xCD9E8D57 into 64-bit products (hi, lo) and
returns (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0); between rounds the key is
bumped by the Weyl constants (0x9E3779B9, 0xBB67AE85).

Dropout mask of this library ("FlashAttention v2" article, §5.1 lists
``dropout_p``; the pages define no random-number scheme, so this is the
scheme this library defines):
  * threshold t = round(256 p) in [0, 255]; an element is kept iff its random
    byte is >= t, so the keep probability is exactly (256 - t) / 256, and kept
    probabilities are scaled by 256 / (256 - t);
  * the byte of element (b, h, query i, key j) is byte (j mod 4) (least
    significant first) of output word (i mod 4) of Philox4x32-10 with counter
    (j div 4, i div 4, h, b) and key (seed mod 2^32, seed div 2^32).
"""

from __future__ import annotations

import numpy as np

M0 = np.uint64(0xD2511F53)
M1 = np.uint64(0xCD9E8D57)
W0 = np.uint32(0x9E3779B9)
W1 = np.uint32(0xBB67AE85)
MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox4x32-10.  Counters are uint32 arrays (broadcast
    together), keys uint32 scalars.  Returns four uint32 arrays."""
    c0, c1, c2, c3 = (np.asarray(x, dtype=np.uint32) for x in (c0, c1, c2, c3))
    c0, c1, c2, c3 = np.broadcast_arrays(c0, c1, c2, c3)
    c0, c1, c2, c3 = (x.astype(np.uint32, copy=True) for x in (c0, c1, c2, c3))
    k0 = np.uint32(k0)
    k1 = np.uint32(k1)
    with np.errstate(over="ignore"):
        for r in range(10):
            if r > 0:
                k0 = np.uint32(k0 + W0)
                k1 = np.uint32(k1 + W1)
            p0 = M0 * c0.astype(np.uint64)
            p1 = M1 * c2.astype(np.uint64)
            hi0 = (p0 >> np.uint64(32)).astype(np.uint32)
            lo0 = (p0 & MASK32).astype(np.uint32)
            hi1 = (p1 >> np.uint64(32)).astype(np.uint32)
            lo1 = (p1 & MASK32).astype(np.uint32)
            c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def dropout_threshold(p: float) -> int:
    """t = round(256 p), the byte threshold; valid for 0 <= p < 255.5/256."""
    t = int(np.floor(p * 256.0 + 0.5))
    if not 0 <= t <= 255:
        raise ValueError("dropout_p out of range")
    return t


def keep_scale(p: float) -> float:
    t = dropout_threshold(p)
    return 256.0 / (256.0 - t)


def random_bytes(b: int, h: int, rows, n_keys: int, seed: int) -> np.ndarray:
    """uint8 [len(rows), n_keys]: the random byte of each (query, key)."""
    rows = np.asarray(rows, dtype=np.int64)
    j = np.arange(n_keys, dtype=np.int64)
    c0 = (j >> 2).astype(np.uint32)[None, :]
    c1 = (rows >> 2).astype(np.uint32)[:, None]
    k0 = np.uint32(seed & 0xFFFFFFFF)
    k1 = np.uint32((seed >> 32) & 0xFFFFFFFF)
    words = philox4x32_10(c0, c1, np.uint32(h), np.uint32(b), k0, k1)
    w = np.stack(words, axis=0)                       # [4, rows, keys]
    word = np.take_along_axis(w, (rows & 3)[None, :, None].repeat(n_keys, axis=2), axis=0)[0]
    shift = ((j & 3) * 8).astype(np.uint32)[None, :]
    return ((word >> shift) & np.uint32(0xFF)).astype(np.uint8)


def keep_mask(b: int, h: int, rows, n_keys: int, p: float, seed: int) -> np.ndarray:
    """Boolean [len(rows), n_keys]: True where the element is kept."""
    t = dropout_threshold(p)
    return random_bytes(b, h, rows, n_keys, seed) >= t

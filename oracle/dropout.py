"""Dropout masks for the oracle: the Philox4x32-10 counter-based generator and the rule that turns
its output into keep/drop decisions. Plain NumPy. TEST INFRASTRUCTURE ONLY (see the package
docstring).

Where dropout sits. "How FlashAttention Actually Works" (hot.atechcom.net), section "The GPU
Memory Wall: HBM vs. SRAM", lists dropout as a pass over the softmax matrix between the softmax
and the product with V. The pages say nothing more, so the plainest reading is taken: inverted
dropout on P, each entry kept with probability 1 - p and then scaled by 1 / (1 - p), zeroed
otherwise; the row's softmax statistics (m, l, lse) are those of the undropped P.

The random draws. Each side implements Philox4x32-10 from its published definition: J. K.
Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3"
(SC'11), section 4 (the Philox S-box: a 4-word counter, a 2-word key, ten rounds of two 32x32->64
multiplications with the round multipliers 0xD2511F53 and 0xCD9E8D57, the key bumped by the Weyl
constants 0x9E3779B9 and 0xBB67AE85 between rounds). A test pins this to the paper's
known-answer vectors.

The mapping from an attention entry to random bits (this package's own definition; the pages
have none). For query head bh (flattened batch * heads index), query row i and key j:
    counter = (j >> 2, i >> 2, bh, offset),   key = (seed mod 2^32, seed >> 32)
    w0..w3  = Philox4x32-10(counter, key)
    byte    = bits [8 (j & 3), 8 (j & 3) + 8) of w_(i & 3)
    keep    = byte >= p8,  with p8 = min(255, floor(256 p + 1/2))
so one Philox call covers a 4 x 4 block of entries. The drop probability is p8 / 256 (p rounded
to a multiple of 1/256), and kept entries are scaled by 256 / (256 - p8), so the expectation of
a dropped entry is exactly the undropped one.
"""

from __future__ import annotations

import numpy as np

__all__ = ["philox4x32_10", "dropout_p8", "keep_scale", "dropout_keep"]

_M0, _M1 = np.uint64(0xD2511F53), np.uint64(0xCD9E8D57)
_W0, _W1 = 0x9E3779B9, 0xBB67AE85
_LO = np.uint64(0xFFFFFFFF)
_SH = np.uint64(32)


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Philox4x32 with 10 rounds on arrays of counters (broadcast together) and one key.

    One round, per the SC'11 paper: (hi0, lo0) = M0 * c0, (hi1, lo1) = M1 * c2 as 64-bit
    products, then (c0, c1, c2, c3) <- (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0); the key is
    bumped by (W0, W1) after each round. Returns four uint32 arrays."""
    c = [np.asarray(x, dtype=np.uint64) & _LO for x in (c0, c1, c2, c3)]
    c = list(np.broadcast_arrays(*c))
    ka, kb = int(k0) & 0xFFFFFFFF, int(k1) & 0xFFFFFFFF
    for _ in range(10):
        p0 = _M0 * c[0]
        p1 = _M1 * c[2]
        c = [(p1 >> _SH) ^ c[1] ^ np.uint64(ka), p1 & _LO,
             (p0 >> _SH) ^ c[3] ^ np.uint64(kb), p0 & _LO]
        ka = (ka + _W0) & 0xFFFFFFFF
        kb = (kb + _W1) & 0xFFFFFFFF
    return tuple(x.astype(np.uint32) for x in c)


def dropout_p8(p: float) -> int:
    """Drop threshold in 1/256 units: min(255, floor(256 p + 1/2)); p in [0, 1)."""
    p = float(np.float32(p))
    if not (0.0 <= p < 1.0):
        raise ValueError("dropout probability must be in [0, 1)")
    return min(255, int(np.floor(256.0 * p + 0.5)))


def keep_scale(p8: int) -> float:
    """Factor applied to kept entries: 1 / (1 - p8/256)."""
    return 256.0 / (256.0 - p8)


def dropout_keep(bh: int, rows, keys, p8: int, seed: int, offset: int) -> np.ndarray:
    """Keep decisions Z [len(rows), len(keys)] (bool) of query head `bh` for the given query
    rows and keys (an int n stands for keys 0 .. n-1), following the mapping in the module
    docstring."""
    i = np.asarray(rows, dtype=np.int64).reshape(-1, 1)
    if np.isscalar(keys) or np.ndim(keys) == 0:
        keys = np.arange(int(keys))
    j = np.asarray(keys, dtype=np.int64).reshape(1, -1)
    n_keys = j.shape[1]
    w = philox4x32_10(j >> 2, i >> 2, np.int64(bh), np.int64(offset), seed & 0xFFFFFFFF,
                      (seed >> 32) & 0xFFFFFFFF)
    sel = np.broadcast_to(i & 3, (i.shape[0], n_keys))
    word = np.choose(sel, w)
    byte = (word >> (8 * (j & 3)).astype(np.uint32)) & np.uint32(0xFF)
    return byte >= np.uint32(p8)

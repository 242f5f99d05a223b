"""Philox4x32-10 counter-based generator and the Gumbel noise drawn from it.

TEST INFRASTRUCTURE: this package is the fp64 CPU oracle.  Only tests/,
__graft_entry__.smoke() and bench.py's CPU-baseline / reference legs may import
it.  The product path never does.

The pages fix no sampling mechanism for T=1 (Domino study notes, gsyq.cn,
§三.2(1) "采样解码（T=1）"; yhxrc.cn article, §六).  This build samples with
Gumbel-max driven by Philox4x32-10 as defined in Salmon, Moraes, Dror and Shaw,
"Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11), §4 (the Philox
S-box: two 32x32->64 multiplies per round, a Weyl sequence on the key).

Noise for request b, 1-based position i, vocabulary index j:
  key     = (seed mod 2^32, seed >> 32)
  counter = (j >> 2, i - 1, b, 0), output word j & 3 -> w
  u       = (2 * (w >> 9) + 1) * 2^-24        (exact in fp32, strictly inside (0, 1))
  g       = -log(-log(u))
"""
from __future__ import annotations

import numpy as np

PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9  # golden ratio
PHILOX_W1 = 0xBB67AE85  # sqrt(3) - 1
_MASK32 = 0xFFFFFFFF


def philox4x32_10(counter, key):
    """One Philox4x32-10 block: four 32-bit counter words, two key words -> four words.

    Plain Python integers; one round maps (x0, x1, x2, x3) to
    (hi(M1*x2) ^ x1 ^ k0, lo(M1*x2), hi(M0*x0) ^ x3 ^ k1, lo(M0*x0)),
    then the key advances by the Weyl constants.
    """
    x0, x1, x2, x3 = (int(c) & _MASK32 for c in counter)
    k0, k1 = (int(k) & _MASK32 for k in key)
    for _ in range(10):
        p0 = PHILOX_M0 * x0
        p1 = PHILOX_M1 * x2
        x0, x1, x2, x3 = ((p1 >> 32) ^ x1 ^ k0, p1 & _MASK32, (p0 >> 32) ^ x3 ^ k1, p0 & _MASK32)
        k0 = (k0 + PHILOX_W0) & _MASK32
        k1 = (k1 + PHILOX_W1) & _MASK32
    return (x0, x1, x2, x3)


def philox4x32_10_np(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox4x32-10 over uint32 numpy arrays (same definition as above)."""
    x0, x1, x2, x3 = (np.asarray(c, dtype=np.uint64) & np.uint64(_MASK32) for c in (c0, c1, c2, c3))
    k0 = np.uint64(int(k0) & _MASK32)
    k1 = np.uint64(int(k1) & _MASK32)
    m = np.uint64(_MASK32)
    s = np.uint64(32)
    for _ in range(10):
        p0 = np.uint64(PHILOX_M0) * x0
        p1 = np.uint64(PHILOX_M1) * x2
        x0, x1, x2, x3 = ((p1 >> s) ^ x1 ^ k0, p1 & m, (p0 >> s) ^ x3 ^ k1, p0 & m)
        k0 = (k0 + np.uint64(PHILOX_W0)) & m
        k1 = (k1 + np.uint64(PHILOX_W1)) & m
    return tuple(x.astype(np.uint32) for x in (x0, x1, x2, x3))


def uniform_from_word(w):
    """Map a 32-bit word to u = (2*(w>>9)+1) * 2^-24 in (0, 1), as fp64 (exact)."""
    w = np.asarray(w, dtype=np.uint64)
    return ((w >> np.uint64(9)).astype(np.float64) * 2.0 + 1.0) * 2.0 ** -24


def gumbel_noise(seed: int, b: int, i: int, V: int) -> np.ndarray:
    """Gumbel noise g[j], j in [0, V), for request b and 1-based position i (fp64)."""
    j = np.arange(V, dtype=np.uint64)
    blocks = (np.arange((V + 3) // 4, dtype=np.uint64))
    words = philox4x32_10_np(blocks, np.full_like(blocks, i - 1), np.full_like(blocks, b),
                             np.zeros_like(blocks), seed & _MASK32, (seed >> 32) & _MASK32)
    w = np.stack(words, axis=1).reshape(-1)[:V]
    assert w.shape[0] == j.shape[0]
    u = uniform_from_word(w)
    return -np.log(-np.log(u))

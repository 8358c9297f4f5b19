"""Philox4x32-10 and the Box-Muller normals drawn from it -- CPU oracle side.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and
bench.py's CPU-baseline leg, never by the product path.

The training recipe draws its initial weights from N(0, 0.02) ("Pretraining
and adapting a language model on a dependency-free stack", §4.1). Those random
numbers cannot be passed in as inputs to gpt2_create (which takes a seed), so
both sides implement one counter-based generator from its published
definition: Philox4x32 with 10 rounds (Salmon, Moraes, Dror, Shaw,
"Parallel random numbers: as easy as 1, 2, 3", SC'11, §3 and Table 2).

Round function on a counter (c0, c1, c2, c3) and key (k0, k1):
    (hi0, lo0) = M0 * c0,  (hi1, lo1) = M1 * c2      (32x32 -> 64-bit products)
    out = (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0)
with multipliers M0 = 0xD2511F53, M1 = 0xCD9E8D57; between rounds the key is
bumped by the Weyl constants (0x9E3779B9, 0xBB67AE85).

Normals: for counter block c of stream ``kind`` the generator is called on
counter (c mod 2^32, c div 2^32, kind, 0) and key (seed mod 2^32, seed div
2^32). Each 32-bit output x becomes u = ((x >> 9) + 0.5) / 2^23, which lies in
(0, 1) and is exact in both fp32 and fp64 (the top 23 bits plus a half need
24 significant bits, the fp32 significand). Box-Muller (G. E. P. Box and M. E.
Muller, Ann. Math. Statist. 29 (1958)) turns (u0, u1) into
r cos(2 pi u1), r sin(2 pi u1) with r = sqrt(-2 ln u0), and likewise (u2, u3);
element 4c + j of the stream takes the j-th of these four normals.
"""
from __future__ import annotations

import numpy as np

M0 = np.uint64(0xD2511F53)
M1 = np.uint64(0xCD9E8D57)
W0 = np.uint32(0x9E3779B9)
W1 = np.uint32(0xBB67AE85)
MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox4x32-10 over uint32 arrays (counters) and scalars (key)."""
    c0 = np.asarray(c0, dtype=np.uint32)
    c1 = np.asarray(c1, dtype=np.uint32)
    c2 = np.asarray(c2, dtype=np.uint32)
    c3 = np.asarray(c3, dtype=np.uint32)
    k0 = np.uint32(k0)
    k1 = np.uint32(k1)
    for r in range(10):
        if r > 0:
            k0 = np.uint32((int(k0) + int(W0)) & 0xFFFFFFFF)
            k1 = np.uint32((int(k1) + int(W1)) & 0xFFFFFFFF)
        p0 = M0 * c0.astype(np.uint64)
        p1 = M1 * c2.astype(np.uint64)
        hi0 = (p0 >> np.uint64(32)).astype(np.uint32)
        lo0 = (p0 & MASK32).astype(np.uint32)
        hi1 = (p1 >> np.uint64(32)).astype(np.uint32)
        lo1 = (p1 & MASK32).astype(np.uint32)
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def uniform_from_bits(x: np.ndarray) -> np.ndarray:
    """Map 32 random bits to (0, 1): ((x >> 9) + 0.5) / 2^23, exact in fp32."""
    return ((x >> np.uint32(9)).astype(np.float64) + 0.5) * (1.0 / 8388608.0)


def normals(kind: int, n: int, seed: int) -> np.ndarray:
    """First ``n`` standard normals of stream ``kind`` for ``seed`` (fp64)."""
    nblk = (n + 3) // 4
    c = np.arange(nblk, dtype=np.uint64)
    c0 = (c & MASK32).astype(np.uint32)
    c1 = (c >> np.uint64(32)).astype(np.uint32)
    c2 = np.full(nblk, kind, dtype=np.uint32)
    c3 = np.zeros(nblk, dtype=np.uint32)
    x0, x1, x2, x3 = philox4x32_10(c0, c1, c2, c3, seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    u0, u1, u2, u3 = (uniform_from_bits(x) for x in (x0, x1, x2, x3))
    r01 = np.sqrt(-2.0 * np.log(u0))
    r23 = np.sqrt(-2.0 * np.log(u2))
    out = np.empty((nblk, 4), dtype=np.float64)
    out[:, 0] = r01 * np.cos(2.0 * np.pi * u1)
    out[:, 1] = r01 * np.sin(2.0 * np.pi * u1)
    out[:, 2] = r23 * np.cos(2.0 * np.pi * u3)
    out[:, 3] = r23 * np.sin(2.0 * np.pi * u3)
    return out.reshape(-1)[:n]

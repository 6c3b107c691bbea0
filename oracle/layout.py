"""Naive reference packer for the FluxBin device weight layout -- TEST INFRASTRUCTURE ONLY.

Written independently from the layout's definition in ``include/fluxbin.h``
(section "Packed sign layout"); it shares no code with the library's packer
and exists so that the tests can require bit-exact agreement with it.

Definition (one branch: nb bases, ncols columns, M rows, sub-vector length mu):
  P  = 32 / nb                 sub-vectors of one base in a unit
  U  = ceil(ncols / (P*mu))    units (column blocks of P*mu columns)
  Ms = ceil(M / 32)            row slabs of 32 rows
  element (k, i, n) with sign +1 sets one bit, -1 (and padding) leaves it 0:
    s, L  = i // 32, i % 32
    jg, t = n // mu, n % mu
    u, j  = jg // P, jg % P
    a     = (k - L // P) mod nb
    q     = a*P + ((j - L) mod P)           visit step of that sub-vector for lane L
  (grouped order, for a branch whose row scales change every gsv < P
   sub-vectors: KG = 32/gsv, NG = P/gsv, m, g = L // gsv, L % gsv,
    kg = k*NG + j // gsv, a = (kg - m) mod KG, q = a*gsv + ((j mod gsv) xor g))
    pos   = q*mu + t
    word  = (s*U + u)*(32*mu) + ((pos // 128)*32 + L)*4 + (pos // 32) % 4
    bit   = pos % 32
"""
from __future__ import annotations

import numpy as np


def branch_geometry(M: int, ncols: int, nb: int, mu: int):
    P = 32 // nb
    U = -(-ncols // (P * mu)) if ncols > 0 else 0
    Ms = -(-M // 32) if M > 0 else 0
    return P, U, Ms


def branch_words(M: int, ncols: int, nb: int, mu: int) -> int:
    P, U, Ms = branch_geometry(M, ncols, nb, mu)
    return Ms * U * 32 * mu


def _positions(M: int, ncols: int, nb: int, mu: int, gsv: int = 0):
    P, U, Ms = branch_geometry(M, ncols, nb, mu)
    k = np.arange(nb, dtype=np.int64)[:, None, None]
    i = np.arange(M, dtype=np.int64)[None, :, None]
    n = np.arange(ncols, dtype=np.int64)[None, None, :]
    s, L = i // 32, i % 32
    jg, t = n // mu, n % mu
    u, j = jg // P, jg % P
    if gsv and gsv < P:
        KG, NG = 32 // gsv, P // gsv
        m, sg = L // gsv, L % gsv
        kg = k * NG + j // gsv
        a = np.mod(kg - m, KG)
        q = a * gsv + np.bitwise_xor(j % gsv, sg)
    else:
        a = np.mod(k - L // P, nb)
        q = a * P + np.mod(j - L, P)
    pos = q * mu + t
    word = (s * U + u) * (32 * mu) + ((pos // 128) * 32 + L) * 4 + (pos // 32) % 4
    bit = pos % 32
    word, bit = np.broadcast_arrays(word, bit)
    return word, bit


def pack_branch(signs: np.ndarray, mu: int, gsv: int = 0) -> np.ndarray:
    """signs int8 [nb][M][ncols] (+-1) -> uint32 words of the device layout
    (gsv: sub-vectors per row-scale group for the grouped visit order)."""
    nb, M, ncols = signs.shape
    total = branch_words(M, ncols, nb, mu)
    out = np.zeros(total, dtype=np.uint64)
    if total == 0:
        return out.astype(np.uint32)
    word, bit = _positions(M, ncols, nb, mu, gsv)
    plus = signs > 0
    # every (word, bit) pair is distinct, so adding the set bits is an OR
    np.add.at(out, word[plus], np.left_shift(np.uint64(1), bit[plus].astype(np.uint64)))
    return out.astype(np.uint32)


def unpack_branch(words: np.ndarray, M: int, ncols: int, nb: int, mu: int, gsv: int = 0) -> np.ndarray:
    """Inverse of pack_branch: uint32 words -> int8 signs [nb][M][ncols]."""
    word, bit = _positions(M, ncols, nb, mu, gsv)
    w = np.asarray(words, dtype=np.uint32)
    bits = (w[word] >> bit.astype(np.uint32)) & 1
    return (bits.astype(np.int8) * 2 - 1).astype(np.int8)

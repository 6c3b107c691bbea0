"""FluxBin decomposition fitting, plain fp64 numpy -- TEST INFRASTRUCTURE ONLY.

Only ``tests/`` and the CPU legs of ``bench.py`` may import this module; the
library's own fitter (``fluxbin_fit`` / ``fluxbin_fit_hybrid`` in
libfluxbin.so) shares no code with it.

What it computes ("FluxBin: Flexible LUT-based Ultra-low-bit LLM Inference by
Algorithm-Kernel Synergy", source-linked summary):

  Section 3 "Quantization" / "Parameter Optimization": W is approximated by
  sum_k diag(r_k) B_k diag(c_k) with B_k in {-1,+1}, the scales and the bases
  chosen to minimise the (weighted) reconstruction error by alternating
  minimisation; for several bases all 2^Kb sign combinations of an element are
  evaluated jointly.
  Appendix A.1: with B and c fixed, the objective separates into one scalar
  least-squares problem per row scale, solved in closed form by setting the
  derivative to zero (and, symmetrically, one per column scale).
  Appendix A.2: with the scales fixed, the error separates over the elements
  of W; an exhaustive search over b in {-1,+1}^Kb per element is globally
  optimal.
  Section 3 "Salient-Aware Hybrid Bases": the salient branch applies the same
  quantisation function, with its own bases and scales, to the residual of the
  global branch on the salient columns.
  Appendix C.2: row scales may be block-wise (one per row per G columns).

Readings where the pages are silent (plainest choices):
  * objective: sum_ij h_j (W_ij - What_ij)^2 with per-column weights h
    (all 1 by default) -- the "weighted least squares" of the summary with the
    weight carried per input column;
  * initialisation: greedy on the residual, base by base: B_k = sign(R)
    (sign(0) = +1), c_k = 1, r_k = the closed-form row scale for c = 1 (the
    weighted mean of |R| over the row or row block), R -= diag(r_k) B_k;
  * one iteration: for every base k in order, with the other bases fixed, the
    row scales of k (closed form, A.1) and then its column scales (closed form);
    then the joint sign search over all elements (A.2);
  * a scale whose denominator is zero is set to 0; among sign combinations with
    equal error the first in the order p = 0 .. 2^Kb - 1 wins (bit k of p set
    means b_k = +1).
"""
from __future__ import annotations

from typing import Optional

import numpy as np


def _row_groups(N: int, G: int) -> np.ndarray:
    """Block index of every column (0 for every column when G == 0)."""
    return (np.arange(N) // G) if G > 0 else np.zeros(N, np.int64)


def _expand_r(r: np.ndarray, N: int, G: int) -> np.ndarray:
    """Row scale of every (row, column): r is [M] (G == 0) or [ng][M]."""
    if G <= 0:
        return np.repeat(r[:, None], N, axis=1)
    return r[_row_groups(N, G), :].T


def base_matrix(B: np.ndarray, r: np.ndarray, c: np.ndarray, G: int) -> np.ndarray:
    """diag(r) B diag(c) of one base (block-wise r when G > 0)."""
    return _expand_r(r, B.shape[1], G) * B.astype(np.float64) * c[None, :]


def reconstruct(signs, r, c, G: int) -> np.ndarray:
    """sum_k diag(r_k) B_k diag(c_k)."""
    out = np.zeros(signs.shape[1:], np.float64)
    for k in range(signs.shape[0]):
        out += base_matrix(signs[k], r[k], c[k], G)
    return out


def objective(W, signs, r, c, G: int, h: Optional[np.ndarray] = None) -> float:
    """sum_ij h_j (W_ij - What_ij)^2."""
    h = np.ones(W.shape[1]) if h is None else np.asarray(h, np.float64)
    E = W - reconstruct(signs, r, c, G)
    return float(np.sum(h[None, :] * E * E))


def row_scale_update(R, Bk, ck, G: int, h) -> np.ndarray:
    """Appendix A.1: for fixed B_k and c_k the best row scale of row i (or of
    block g of row i) is sum_j h_j R_ij B_ij c_j / sum_j h_j c_j^2 over the
    row (block)."""
    M, N = R.shape
    num_el = h[None, :] * R * Bk * ck[None, :]
    den_el = h * ck * ck
    if G <= 0:
        num = num_el.sum(axis=1)
        den = den_el.sum()
        return num / den if den != 0 else np.zeros(M)
    ng = (N + G - 1) // G
    out = np.zeros((ng, M))
    for g in range(ng):
        sl = slice(g * G, min(N, (g + 1) * G))
        den = den_el[sl].sum()
        out[g] = num_el[:, sl].sum(axis=1) / den if den != 0 else 0.0
    return out


def col_scale_update(R, Bk, rk, G: int) -> np.ndarray:
    """The symmetric closed form for the column scales with B_k and r_k fixed:
    c_j = sum_i R_ij B_ij r_i(j) / sum_i r_i(j)^2 (the column weight h_j is a
    common factor of column j and cancels)."""
    Rx = _expand_r(rk, R.shape[1], G)
    num = (R * Bk * Rx).sum(axis=0)
    den = (Rx * Rx).sum(axis=0)
    out = np.zeros(R.shape[1])
    nz = den != 0
    out[nz] = num[nz] / den[nz]
    return out


def sign_search(W, r, c, G: int) -> np.ndarray:
    """Appendix A.2: every element takes the b in {-1,+1}^nb that minimises
    (W_ij - sum_k r_k(i,j) c_k[j] b_k)^2, all 2^nb combinations evaluated."""
    nb = len(r)
    M, N = W.shape
    S = np.stack([_expand_r(r[k], N, G) * c[k][None, :] for k in range(nb)])   # [nb][M][N]
    best_err = np.full((M, N), np.inf)
    best_p = np.zeros((M, N), np.int64)
    for p in range(1 << nb):
        approx = np.zeros((M, N))
        for k in range(nb):
            approx += S[k] if (p >> k) & 1 else -S[k]
        err = (W - approx) ** 2
        better = err < best_err
        best_err = np.where(better, err, best_err)
        best_p = np.where(better, p, best_p)
    return np.stack([np.where((best_p >> k) & 1, 1, -1).astype(np.int8) for k in range(nb)])


def init_greedy(W, nb: int, G: int, h):
    """Greedy residual start: B_k = sign(R), c_k = 1, r_k by A.1 with c = 1."""
    M, N = W.shape
    R = W.copy()
    signs, rs, cs = [], [], []
    for _ in range(nb):
        Bk = np.where(R >= 0, 1, -1).astype(np.int8)
        ck = np.ones(N)
        rk = row_scale_update(R, Bk, ck, G, h)
        R = R - base_matrix(Bk, rk, ck, G)
        signs.append(Bk)
        rs.append(rk)
        cs.append(ck)
    return np.stack(signs), rs, cs


def fit(W, nb: int, G: int = 0, iters: int = 10, h: Optional[np.ndarray] = None, history: bool = False):
    """Alternating minimisation: returns (signs [nb][M][N] int8, r list of [M]
    or [ng][M], c list of [N]) and, with history, the objective after the
    start and after every iteration."""
    W = np.asarray(W, np.float64)
    h = np.ones(W.shape[1]) if h is None else np.asarray(h, np.float64)
    signs, r, c = init_greedy(W, nb, G, h)
    hist = [objective(W, signs, r, c, G, h)]
    for _ in range(iters):
        for k in range(nb):
            Rk = W.copy()
            for l in range(nb):
                if l != k:
                    Rk -= base_matrix(signs[l], r[l], c[l], G)
            Bk = signs[k].astype(np.float64)
            r[k] = row_scale_update(Rk, Bk, c[k], G, h)
            c[k] = col_scale_update(Rk, Bk, r[k], G)
        signs = sign_search(W, r, c, G)
        hist.append(objective(W, signs, r, c, G, h))
    if history:
        return signs, r, c, hist
    return signs, r, c


def fit_hybrid(W, sal_idx, Kb: int, Ks: int, G: int = 0, Gs: int = 0, iters: int = 10,
               h: Optional[np.ndarray] = None):
    """Global bases on W, then the salient refinement: the same fit on the
    global residual gathered at the salient columns (a dense M x n_sal matrix,
    the Virtual Columnar Mapping layout), with its own bases and scales."""
    W = np.asarray(W, np.float64)
    h = np.ones(W.shape[1]) if h is None else np.asarray(h, np.float64)
    signs, r, c = fit(W, Kb, G, iters, h)
    sal_idx = np.asarray(sal_idx, np.int64)
    if Ks == 0 or sal_idx.size == 0:
        return (signs, r, c), None
    R = (W - reconstruct(signs, r, c, G))[:, sal_idx]
    s_signs, s_r, s_c = fit(R, Ks, Gs, iters, h[sal_idx])
    return (signs, r, c), (s_signs, s_r, s_c)

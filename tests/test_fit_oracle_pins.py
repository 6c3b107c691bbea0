"""Pins of the oracle's decomposition fitting (oracle/fit.py) to what the
pages and the mathematics fix, independent of the oracle itself.

FluxBin summary: Section 3 "Parameter Optimization" (alternating
minimisation, joint sign search over 2^Kb combinations), Appendix A.1
(closed-form row and column scales), Appendix A.2 (element-wise exhaustive
search is globally optimal for fixed scales), Section 3 "Salient-Aware
Hybrid Bases" (the salient branch fits the residual on the salient columns).

  * exact recovery: a one-base W = diag(r) B diag(c) (per-row or block-wise
    r) is reproduced to fp64 rounding, with B itself;
  * the scale updates equal weighted least squares solved by a library
    routine (numpy lstsq) one row / one column at a time;
  * the sign step is the global minimum over every sign tensor, by brute
    force on tiny shapes;
  * the objective never increases over the iterations;
  * the salient refinement leaves the columns outside S untouched and never
    raises the error.
Planted mistakes in copies of the steps are each caught by one of them.
"""
import itertools

import numpy as np
import pytest

from oracle import fit as F


def _rng(seed):
    return np.random.default_rng(seed)


def _signs(rng, shape):
    return np.where(rng.random(shape) < 0.5, 1, -1).astype(np.int8)


def _aniso(rng, M, N):
    return (np.exp(0.5 * rng.standard_normal(M))[:, None] * np.exp(0.5 * rng.standard_normal(N))[None, :]
            * rng.standard_normal((M, N)))


# ---------------------------------------------------------------------------
# pins, each taking the step (or the whole fit) under test
# ---------------------------------------------------------------------------

def pin_exact_one_base(fit):
    rng = _rng(3)
    M, N = 23, 70
    for G in (0, 16):
        B = _signs(rng, (M, N))
        c = np.exp(0.4 * rng.standard_normal(N))
        r = np.exp(0.4 * rng.standard_normal((M,) if G == 0 else (-(-N // G), M)))
        W = F.base_matrix(B, r, c, G) if G else r[:, None] * B * c[None, :]
        s, rr, cc = fit(W, 1, G, 2)
        What = F.reconstruct(s, rr, cc, G)
        assert np.array_equal(s[0], B)
        assert np.linalg.norm(What - W) <= 1e-13 * np.linalg.norm(W)


def pin_row_scale_is_weighted_lstsq(row_update):
    rng = _rng(4)
    M, N = 9, 40
    for G in (0, 8):
        R = rng.standard_normal((M, N))
        Bk = _signs(rng, (M, N)).astype(np.float64)
        ck = np.exp(0.3 * rng.standard_normal(N))
        h = rng.random(N) + 0.1
        got = row_update(R, Bk, ck, G, h)
        groups = [np.arange(N)] if G == 0 else [np.arange(g * G, min(N, (g + 1) * G)) for g in range(-(-N // G))]
        for i in range(M):
            for g, cols in enumerate(groups):
                a = (np.sqrt(h[cols]) * Bk[i, cols] * ck[cols])[:, None]
                want = np.linalg.lstsq(a, np.sqrt(h[cols]) * R[i, cols], rcond=None)[0][0]
                have = got[i] if G == 0 else got[g, i]
                assert abs(have - want) <= 1e-12 * max(1.0, abs(want))


def pin_col_scale_is_lstsq(col_update):
    rng = _rng(5)
    M, N = 30, 11
    for G in (0, 4):
        R = rng.standard_normal((M, N))
        Bk = _signs(rng, (M, N)).astype(np.float64)
        rk = np.exp(0.3 * rng.standard_normal((M,) if G == 0 else (-(-N // G), M)))
        got = col_update(R, Bk, rk, G)
        for j in range(N):
            rcol = rk if G == 0 else rk[j // G]
            want = np.linalg.lstsq((Bk[:, j] * rcol)[:, None], R[:, j], rcond=None)[0][0]
            assert abs(got[j] - want) <= 1e-12 * max(1.0, abs(want))


def pin_sign_search_global(search):
    rng = _rng(6)
    for (M, N, nb) in ((2, 3, 2), (1, 3, 3), (3, 2, 2)):
        W = rng.standard_normal((M, N))
        r = [np.exp(0.5 * rng.standard_normal(M)) for _ in range(nb)]
        c = [np.exp(0.5 * rng.standard_normal(N)) for _ in range(nb)]
        got = search(W, r, c, 0)
        got_err = F.objective(W, got, r, c, 0)
        best = np.inf
        for bits in itertools.product((-1, 1), repeat=nb * M * N):
            s = np.array(bits, np.int8).reshape(nb, M, N)
            best = min(best, F.objective(W, s, r, c, 0))
        assert got_err <= best * (1 + 1e-12) + 1e-300


def pin_monotone(fit_hist):
    rng = _rng(7)
    for nb, G in ((1, 0), (2, 0), (3, 16), (2, 8)):
        W = _aniso(rng, 31, 48)
        h = rng.random(48) + 0.2
        hist = fit_hist(W, nb, G, 6, h)
        for a, b in zip(hist, hist[1:]):
            assert b <= a * (1 + 1e-12)
        assert hist[-1] < hist[0]


def fit_hist_oracle(W, nb, G, iters, h):
    return F.fit(W, nb, G, iters, h, history=True)[3]


# ---------------------------------------------------------------------------
# the oracle against its pins
# ---------------------------------------------------------------------------

def test_exact_one_base():
    pin_exact_one_base(F.fit)


def test_row_scale_is_weighted_lstsq():
    pin_row_scale_is_weighted_lstsq(F.row_scale_update)


def test_col_scale_is_lstsq():
    pin_col_scale_is_lstsq(F.col_scale_update)


def test_sign_search_global():
    pin_sign_search_global(F.sign_search)


def test_objective_monotone():
    pin_monotone(fit_hist_oracle)


def test_hybrid_refines_only_salient_columns():
    rng = _rng(8)
    M, N = 40, 96
    W = _aniso(rng, M, N)
    S = np.sort(rng.choice(N, 12, replace=False))
    (gs, gr, gc), sal = F.fit_hybrid(W, S, 2, 2, G=32, Gs=4, iters=5)
    glob = F.reconstruct(gs, gr, gc, 32)
    ss, sr, sc = sal
    full = glob.copy()
    full[:, S] += F.reconstruct(ss, sr, sc, 4)
    outside = np.setdiff1d(np.arange(N), S)
    assert np.array_equal(full[:, outside], glob[:, outside])
    assert np.sum((W - full) ** 2) < np.sum((W - glob) ** 2)
    # the global branch is exactly the stand-alone fit
    s2, r2, c2 = F.fit(W, 2, 32, 5)
    assert np.array_equal(s2, gs) and all(np.array_equal(a, b) for a, b in zip(r2, gr))


# ---------------------------------------------------------------------------
# planted mistakes, each caught by a pin
# ---------------------------------------------------------------------------

def _row_update_unweighted(R, Bk, ck, G, h):
    return F.row_scale_update(R, Bk, ck, G, np.ones_like(h))


def _col_update_linear_den(R, Bk, rk, G):
    Rx = F._expand_r(rk, R.shape[1], G)
    return (R * Bk * Rx).sum(axis=0) / np.abs(Rx).sum(axis=0)


def _sign_search_greedy(W, r, c, G):
    # base by base on the residual instead of jointly
    out, R = [], W.copy()
    for k in range(len(r)):
        S = F._expand_r(r[k], W.shape[1], G) * c[k][None, :]
        b = np.where(R >= 0, 1, -1).astype(np.int8)
        out.append(b)
        R = R - b * S
    return np.stack(out)


def _row_den_linear(R, Bk, ck, G, h):
    """Row closed form dividing by sum_j h_j c_j instead of sum_j h_j c_j^2."""
    M, N = R.shape
    num_el = h[None, :] * R * Bk * ck[None, :]
    den_el = h * ck
    if G <= 0:
        return num_el.sum(axis=1) / den_el.sum()
    ng = -(-N // G)
    return np.stack([num_el[:, g * G:(g + 1) * G].sum(axis=1) / den_el[g * G:(g + 1) * G].sum() for g in range(ng)])


def _fit_col_update_without_signs(W, nb, G=0, iters=10, h=None):
    """The whole fit with the column closed form leaving out the base's signs."""
    orig = F.col_scale_update

    def wrong(R, Bk, rk, G_):
        return orig(R, np.ones_like(Bk), rk, G_)

    F.col_scale_update = wrong
    try:
        return F.fit(W, nb, G, iters, h)
    finally:
        F.col_scale_update = orig


@pytest.mark.parametrize("pin,broken", [
    (pin_row_scale_is_weighted_lstsq, _row_update_unweighted),
    (pin_col_scale_is_lstsq, _col_update_linear_den),
    (pin_sign_search_global, _sign_search_greedy),
    (pin_row_scale_is_weighted_lstsq, _row_den_linear),
    (pin_exact_one_base, _fit_col_update_without_signs),
], ids=["unweighted_rows", "linear_col_denominator", "greedy_signs", "row_denominator_linear",
        "col_update_without_signs"])
def test_planted_fit_mistake_is_caught(pin, broken):
    with pytest.raises(AssertionError):
        pin(broken)

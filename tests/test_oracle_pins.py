"""Pins for the fp64 oracle: closed forms, invariants, library routines on
special cases and brute force, each chosen so that a plausible mistake (a
dropped term, a wrong sign or index, a scale on the wrong side) fails one.

Every pin takes the function under test as an argument; the same pins are
run against deliberately broken copies (planted mistakes, on the CPU) to show
that each mistake is caught.
"""
import dataclasses
import itertools

import numpy as np
import pytest

import oracle
from lut_binary_basis_b200.synth import LayerSpec, make_exact_layer, make_exact_x, make_layer, make_x


def spec_of(M, N, Kb, Ks=0, n_sal=0, mu=4, G=0, Gs=0, per_group=0):
    return LayerSpec("pin", M, N, Kb, Ks, n_sal, mu, row_scale_group=G, sal_scale_group=Gs,
                     sal_per_group=per_group)


def sub_bases(d, ks):
    """The same layer restricted to global bases ``ks`` and no salient branch."""
    sp = dataclasses.replace(d.spec, Kb=len(ks), Ks=0, n_sal=0, sal_scale_group=0, sal_per_group=0)
    return dataclasses.replace(d, spec=sp, signs=d.signs[ks], r=d.r[ks], c=d.c[ks],
                               sal_idx=np.zeros(0, np.int32), sal_signs=np.zeros((0, sp.M, 0), np.int8),
                               rs=np.zeros((0, sp.M), np.float16), cs=np.zeros((0, 0), np.float16))


def only_salient(d):
    """The salient branch alone (global bases with zero column scales)."""
    return dataclasses.replace(d, c=np.zeros_like(d.c))


# ----------------------------------------------------------------------------
# Pins on the layer function: linear(layer, x) -> y [B][M]
# ----------------------------------------------------------------------------

def pin_sign_gemv(linear):
    """Kb = 1, unit scales, no salient branch: y = B x, an integer matmul."""
    sp = spec_of(37, 53, 1)
    d = make_exact_layer(sp, [1], unit_scales=True)
    x = make_exact_x(sp, 3, [2])
    ref = (d.signs[0].astype(np.int64) @ x.astype(np.int64).T).T
    assert np.array_equal(linear(d, x), ref.astype(np.float64))


def pin_row_scale_per_row(linear):
    """Multiplying row i's scales by alpha_i multiplies y[:, i] by alpha_i."""
    for G in (0, 8):
        sp = spec_of(19, 24, 2, G=G)
        d = make_exact_layer(sp, [3])
        x = make_exact_x(sp, 2, [4])
        alpha = np.array([0.5, 1.0, 2.0, 4.0], np.float16)[np.arange(sp.M) % 4]
        d2 = dataclasses.replace(d, r=(d.r * alpha).astype(np.float16))
        assert np.array_equal(linear(d2, x), linear(d, x) * alpha.astype(np.float64)[None, :])


def pin_col_scale_per_col(linear):
    """Scaling column j of every base's column scale equals scaling x[:, j]."""
    sp = spec_of(17, 29, 2)
    d = make_exact_layer(sp, [5])
    x = make_exact_x(sp, 2, [6])
    beta = np.array([0.5, 2.0, 1.0], np.float16)[np.arange(sp.N) % 3]
    d2 = dataclasses.replace(d, c=(d.c * beta).astype(np.float16))
    assert np.array_equal(linear(d2, x), linear(d, (x * beta).astype(np.float16)))


def pin_base_additivity(linear):
    """Bases add: y(all bases) = sum over k of y(base k alone) (+ the salient branch)."""
    sp = spec_of(21, 40, 3, Ks=1, n_sal=7)
    d = make_exact_layer(sp, [7])
    x = make_exact_x(sp, 2, [8])
    parts = sum(linear(sub_bases(d, [k]), x) for k in range(3)) + linear(only_salient(d), x)
    assert np.array_equal(linear(d, x), parts)


def pin_salient_scatter(linear):
    """Virtual Columnar Mapping is a re-layout: the salient branch equals extra
    global bases whose signs and column scales are zero outside S."""
    for Ks in (1, 2):
        sp = spec_of(23, 41, 2, Ks=Ks, n_sal=9)
        d = make_exact_layer(sp, [9, Ks])
        x = make_exact_x(sp, 3, [10])
        S = d.sal_idx
        ext_signs = np.zeros((Ks, sp.M, sp.N), np.int8)
        ext_signs[:, :, S] = d.sal_signs
        ext_c = np.zeros((Ks, sp.N), np.float16)
        ext_c[:, S] = d.cs
        base = sub_bases(d, list(range(2)))
        sp2 = dataclasses.replace(base.spec, Kb=2 + Ks)
        d2 = dataclasses.replace(base, spec=sp2, signs=np.concatenate([d.signs, ext_signs]),
                                 r=np.concatenate([d.r, d.rs]), c=np.concatenate([d.c, ext_c]))
        assert np.array_equal(linear(d, x), linear(d2, x))


def pin_salient_permutation(linear):
    """Listing the salient columns in another order (with their signs and
    scales) leaves y unchanged."""
    sp = spec_of(13, 30, 1, Ks=2, n_sal=11)
    d = make_exact_layer(sp, [11])
    x = make_exact_x(sp, 2, [12])
    perm = np.random.default_rng(0).permutation(sp.n_sal)
    d2 = dataclasses.replace(d, sal_idx=d.sal_idx[perm], sal_signs=d.sal_signs[:, :, perm], cs=d.cs[:, perm])
    assert np.array_equal(linear(d, x), linear(d2, x))


def pin_linearity(linear):
    """y(x1 + x2) = y(x1) + y(x2)."""
    sp = spec_of(15, 33, 2, Ks=1, n_sal=5)
    d = make_exact_layer(sp, [13])
    x1 = make_exact_x(sp, 2, [14], -4, 4)
    x2 = make_exact_x(sp, 2, [15], -4, 4)
    assert np.array_equal(linear(d, (x1 + x2).astype(np.float16)), linear(d, x1) + linear(d, x2))


def pin_blockwise_row_scales(linear):
    """Block-wise row scales: (a) equal scales in every block reproduce the
    per-row layer; (b) doubling block g's scales adds block g's share once
    more, and block g's share is y of x masked to that block."""
    sp = spec_of(11, 32, 2, G=8)
    d = make_exact_layer(sp, [16])
    x = make_exact_x(sp, 2, [17])
    per_row = dataclasses.replace(d, spec=dataclasses.replace(sp, row_scale_group=0), r=d.r[:, 0, :])
    flat = dataclasses.replace(d, r=np.repeat(d.r[:, :1, :], d.r.shape[1], axis=1))
    assert np.array_equal(linear(flat, x), linear(per_row, x))
    g = 2
    r2 = d.r.copy()
    r2[:, g, :] *= 2
    mask = np.zeros(sp.N, np.float16)
    mask[g * 8:(g + 1) * 8] = 1
    assert np.array_equal(linear(dataclasses.replace(d, r=r2), x),
                          linear(d, x) + linear(d, (x * mask).astype(np.float16)))


def pin_blockwise_salient_scales(linear):
    """Salient row scales per block of s salient columns: doubling block g's
    salient scales adds once more the salient share of that block."""
    sp = spec_of(9, 40, 1, Ks=2, n_sal=12, Gs=4)
    d = make_exact_layer(sp, [18])
    x = make_exact_x(sp, 2, [19])
    g = 1
    rs2 = d.rs.copy()
    rs2[:, g, :] *= 2
    mask = np.zeros(sp.N, np.float16)
    mask[d.sal_idx[g * 4:(g + 1) * 4]] = 1
    sal_only = only_salient(d)
    assert np.array_equal(linear(dataclasses.replace(d, rs=rs2), x),
                          linear(d, x) + linear(sal_only, (x * mask).astype(np.float16)))


PINS = [pin_sign_gemv, pin_row_scale_per_row, pin_col_scale_per_col, pin_base_additivity,
        pin_salient_scatter, pin_salient_permutation, pin_linearity, pin_blockwise_row_scales,
        pin_blockwise_salient_scales]


def oracle_linear(d, x):
    return oracle.linear(d, x)


def oracle_lut8(d, x):
    # the LUT form needs whole sub-vectors inside every scale block
    return oracle.lut_linear(d, x, mu=4 if (d.spec.row_scale_group or d.spec.sal_scale_group) else 8)


def oracle_lut_sym(d, x):
    return oracle.lut_linear(d, x, mu=4, sym=True)


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
@pytest.mark.parametrize("fn", [oracle_linear, oracle_lut8, oracle_lut_sym], ids=["definition", "lut", "lut_sym"])
def test_oracle_pins(pin, fn):
    pin(fn)


# ----------------------------------------------------------------------------
# Planted mistakes: each broken copy of the definition must fail some pin.
# ----------------------------------------------------------------------------

def broken_linear(mistake):
    def f(d, x):
        sp = d.spec
        M, N = sp.M, sp.N
        Kb = d.signs.shape[0]
        W = np.zeros((M, N))
        nk = Kb - 1 if mistake == "drop_last_base" else Kb
        for k in range(nk):
            s = d.signs[k].astype(np.float64)
            if mistake == "sign_flip":
                s = -s
            ck = d.c[(k + 1) % Kb if mistake == "base_mix" else k].astype(np.float64)
            if mistake == "col_index":
                ck = ck[::-1]
            if sp.row_scale_group:
                gidx = np.arange(N) // sp.row_scale_group
                if mistake == "block_index":
                    gidx = (gidx + 1) % d.r.shape[1]
                rk = d.r[k].astype(np.float64)[gidx, :].T
            elif mistake == "row_by_col":
                rk = d.r[k].astype(np.float64)[np.arange(N) % M][None, :]
            else:
                rk = d.r[k].astype(np.float64)[:, None]
            W += rk * s * ck[None, :]
        if mistake != "drop_salient" and d.sal_idx.size:
            for k in range(d.sal_signs.shape[0]):
                for t, j in enumerate(d.sal_idx):
                    col = (j + 1) % N if mistake == "salient_shift" else j
                    if sp.sal_scale_group:
                        gg = t // sp.sal_scale_group
                        if mistake == "sal_block_index":
                            gg = (gg + 1) % d.rs.shape[1]
                        rr = d.rs[k, gg].astype(np.float64)
                    else:
                        rr = d.rs[k].astype(np.float64)
                    cc = d.c[0, j] if mistake == "salient_global_c" else d.cs[k, t]
                    W[:, col] += rr * d.sal_signs[k, :, t] * float(cc)
        return x.astype(np.float64) @ W.T
    return f


MISTAKES = ["drop_last_base", "sign_flip", "base_mix", "col_index", "block_index", "row_by_col",
            "drop_salient", "salient_shift", "sal_block_index", "salient_global_c"]


def test_unbroken_copy_passes_pins():
    for pin in PINS:
        pin(broken_linear(None))


@pytest.mark.parametrize("mistake", MISTAKES)
def test_planted_mistake_is_caught(mistake):
    caught = []
    for pin in PINS:
        try:
            pin(broken_linear(mistake))
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {mistake!r}"


# ----------------------------------------------------------------------------
# Pins on the table functions
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("mu", range(1, 9))
def test_lut_table_brute_force(mu):
    """Every sign vector s in {-1,+1}^mu, enumerated independently, indexes
    the entry whose bit t is (s_t > 0); that entry is the dot product s . v."""
    v = np.random.default_rng(mu).integers(-50, 50, size=mu).astype(np.float64) / 4
    T = oracle.lut_table(v, mu)
    for s in itertools.product((-1, 1), repeat=mu):
        p = sum(1 << t for t in range(mu) if s[t] > 0)
        assert T[p] == float(np.dot(np.array(s, np.float64), v))


def test_lut_mu1_is_direct_multiply():
    """mu = 1: the table is (-v, +v), so a lookup is the multiply by +-1."""
    for v in (3.25, -0.5, 0.0):
        assert list(oracle.lut_table([v], 1)) == [-v, v]


@pytest.mark.parametrize("mu", [1, 2, 4, 8])
def test_lut_symmetry(mu):
    """T[~p] = -T[p], and the half table plus that rule gives the full table."""
    v = np.random.default_rng(10 + mu).standard_normal(mu)
    T = oracle.lut_table(v, mu)
    mask = (1 << mu) - 1
    for p in range(1 << mu):
        assert T[(~p) & mask] == -T[p]
    Th = oracle.lut_table_sym(v, mu)
    assert Th.size == 1 << (mu - 1)
    assert [oracle.lut_lookup_sym(Th, mu, p) for p in range(1 << mu)] == list(T)


@pytest.mark.parametrize("mu,sym", [(1, False), (2, False), (4, False), (2, True), (4, True)])
def test_lut_form_brute_force_all_sign_matrices(mu, sym):
    """Over all 2^8 sign matrices of a 2 x 4 layer, the LUT evaluation equals
    the definition exactly."""
    sp = spec_of(2, 4, 1)
    d = make_exact_layer(sp, [20])
    x = make_exact_x(sp, 2, [21])
    for bits in range(1 << 8):
        s = np.array([1 if (bits >> e) & 1 else -1 for e in range(8)], np.int8).reshape(1, 2, 4)
        dd = dataclasses.replace(d, signs=s)
        assert np.array_equal(oracle.lut_linear(dd, x, mu=mu, sym=sym), oracle.linear(dd, x))


@pytest.mark.parametrize("mu", [4, 8])
def test_lut_form_random_layers(mu):
    """Random fp16 layers with a salient branch and block-wise scales: the
    LUT evaluation (full and symmetric tables) agrees with the definition to
    fp64 rounding."""
    cases = [spec_of(70, 300, 2, Ks=1, n_sal=15), spec_of(33, 256, 1, Ks=2, n_sal=32, G=64, Gs=16),
             spec_of(40, 129, 4, Ks=1, n_sal=3)]
    for i, sp in enumerate(cases):
        d = make_layer(sp, [30, i])
        x = make_x(sp, 3, [31, i])
        ref = oracle.linear(d, x)
        scale = np.abs(ref).max() + 1
        for sym in (False, True):
            got = oracle.lut_linear(d, x, mu=mu, sym=sym)
            assert np.max(np.abs(got - ref)) <= 1e-12 * scale


def test_row_subsets_match_full():
    """Evaluating selected rows gives the same values as the full output."""
    sp = spec_of(64, 96, 2, Ks=1, n_sal=10)
    d = make_layer(sp, [40])
    x = make_x(sp, 2, [41])
    full = oracle.linear(d, x)
    rows = [63, 0, 17, 17, 40]
    assert np.array_equal(oracle.linear(d, x, rows=rows), full[:, rows])


def test_zero_batch_and_zero_rows():
    sp = spec_of(8, 16, 1)
    d = make_layer(sp, [42])
    assert oracle.linear(d, np.zeros((0, 16), np.float16)).shape == (0, 8)
    assert oracle.linear(d, make_x(sp, 1, [43]), rows=[]).shape == (1, 0)


def oracle_rebuild_then_gemv(d, x):
    return oracle.gemv_rows(oracle.rebuild_rows(d), x)


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_rebuild_then_gemv_pins(pin):
    """The CPU baseline's two timed halves (rows of W rebuilt in fp64, then the
    GEMV on them) satisfy the same closed forms and invariants."""
    pin(oracle_rebuild_then_gemv)


def test_rebuilt_rows_are_columns_of_the_layer_map():
    """Column j of the rebuilt W is the layer's response to the unit vector
    e_j, and a subset of rows is the same rows of the full rebuild."""
    d = make_layer(spec_of(37, 50, 2, 2, 9, G=10, Gs=3), [41])
    W = oracle.rebuild_rows(d)
    E = np.eye(50, dtype=np.float16)
    assert np.array_equal(W.T, oracle.linear(d, E))
    rows = [36, 0, 17]
    assert np.array_equal(oracle.rebuild_rows(d, rows), W[rows])

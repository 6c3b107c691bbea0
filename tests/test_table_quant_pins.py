"""Pins of the oracle's table quantisation (LUT Tensor Core notes, Section
3.1.3: the precomputed table entries are stored in a lower precision, fp16 or
INT8 with a per-table scale).

  * fp16 rounding equals numpy's float16 conversion (round to nearest, ties
    to even) on normal, subnormal, tie and overflow values;
  * the INT8 quantiser picks, for every entry, the code in [-127, 127] that
    is nearest to the entry in units of s = max|T| / 127 (brute force over all
    255 codes, ties to the even code);
  * a layer evaluated with quantised tables equals the sum of the quantised
    table entries its sign patterns select (tables from the brute-force
    definition, quantised with numpy), and stays within the closed-form error
    bounds of the quantisation (fp16: 2^-11 of every entry used; INT8: half a
    scale step per entry used).
Planted mistakes (ties away from zero, a 128-level scale, truncation) fail
these pins.
"""
import numpy as np
import pytest

import oracle
from lut_binary_basis_b200.synth import LayerSpec, make_layer, make_x


def _values(seed=0):
    g = np.random.default_rng(seed)
    v = np.concatenate([g.standard_normal(2000) * 10.0 ** g.integers(-8, 5, 2000),
                        g.uniform(-7e-5, 7e-5, 500),                 # subnormal range
                        np.array([65519.0, 65520.0, -70000.0, 0.0, -0.0, 6.1e-5, 2.0 ** -24, 2.0 ** -25,
                                  3 * 2.0 ** -25])])
    # exact ties between consecutive fp16 values in several binades
    ties = []
    for e in (-20, -14, -3, 0, 5, 14):
        ulp = 2.0 ** (max(e, -14) - 10)
        for k in (1, 2, 3, 1022, 1023):
            ties.append((2.0 ** e if e >= -14 else 0.0) + (k + 0.5) * ulp)
    return np.concatenate([v, np.array(ties), -np.array(ties)])


def pin_fp16(round16):
    for v in _values():
        with np.errstate(over="ignore"):
            want = float(np.float16(v))
        got = round16(float(v))
        assert (np.isinf(want) and got == want) or got == want, (v, got, want)


def pin_int8(quant):
    g = np.random.default_rng(1)
    for trial in range(40):
        T = g.standard_normal(g.choice([16, 128, 256])) * 10.0 ** g.integers(-3, 4)
        if trial == 0:
            T[:] = 0.0
        Tq, s = quant(T)
        m = np.max(np.abs(T))
        if m == 0:
            assert s == 0 and np.all(Tq == 0)
            continue
        assert s == pytest.approx(m / 127, rel=1e-15)
        codes = np.arange(-127, 128)
        for t, tq in zip(T, Tq):
            d = np.abs(t - codes * s)
            best = codes[d == d.min()]
            want = best[0] if best.size == 1 else best[best % 2 == 0][0]
            assert tq == want * s


def test_fp16_rounding_matches_numpy():
    pin_fp16(oracle.round_fp16)


def test_int8_quantiser_brute_force():
    pin_int8(oracle.quantize_table_int8)


@pytest.mark.parametrize("mu", [4, 8])
def test_quantised_tables_equal_selected_entries(mu):
    spec = LayerSpec("q", 5, 2 * mu + 3, 2, 1, 3, mu)
    d = make_layer(spec, [71, mu])
    x = make_x(spec, 2, [72, mu])
    for mode in ("fp16", "int8"):
        got = oracle.lut_linear(d, x, mu=mu, tables=mode)
        want = np.zeros_like(got)
        xd = x.astype(np.float64)
        for b in range(x.shape[0]):
            for br, (signs, r, c, cols) in enumerate(((d.signs, d.r, d.c, np.arange(spec.N)),
                                                      (d.sal_signs, d.rs, d.cs, d.sal_idx))):
                ncols = len(cols)
                for k in range(signs.shape[0]):
                    for j in range(-(-ncols // mu)):
                        v = np.array([c[k][j * mu + t] * xd[b][cols[j * mu + t]] if j * mu + t < ncols else 0.0
                                      for t in range(mu)], np.float64)
                        pats = np.arange(1 << mu)
                        T = np.array([sum(v[t] if (p >> t) & 1 else -v[t] for t in range(mu)) for p in pats])
                        if mode == "fp16":
                            T = T.astype(np.float16).astype(np.float64)
                        else:
                            s = np.max(np.abs(T)) / 127
                            T = np.rint(T / s) * s if s > 0 else T
                        for i in range(spec.M):
                            p = sum(1 << t for t in range(mu) if j * mu + t < ncols and signs[k][i][j * mu + t] > 0)
                            want[b][i] += float(r[k][i]) * T[p]
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12), mode


def test_quantisation_error_bounds():
    spec = LayerSpec("qb", 64, 512, 2, 2, 40, 8)
    d = make_layer(spec, [73])
    x = make_x(spec, 1, [74])
    exact = oracle.lut_linear(d, x, mu=8)
    # |T| of every entry used is at most the sum of |v| of its sub-vector, so
    # per row: fp16 error <= 2^-11 * sum_k |r_k| sum_j sum_t |v_{k,j,t}|
    cols = np.arange(spec.N)
    bound16 = np.zeros(spec.M)
    for signs, r, c, cc in ((d.signs, d.r, d.c, cols), (d.sal_signs, d.rs, d.cs, d.sal_idx)):
        for k in range(signs.shape[0]):
            bound16 += np.abs(r[k].astype(np.float64)) * np.sum(np.abs(c[k].astype(np.float64) *
                                                                      x[0][cc].astype(np.float64)))
    err16 = np.abs(oracle.lut_linear(d, x, mu=8, tables="fp16") - exact)[0]
    assert np.all(err16 <= 2.0 ** -11 * bound16)
    # INT8: half a step (max|T|/127/2 <= sum|v|/254) per table used
    err8 = np.abs(oracle.lut_linear(d, x, mu=8, tables="int8") - exact)[0]
    assert np.all(err8 <= bound16 / 254 + 1e-12)
    assert np.max(err8) > np.max(err16)


# planted mistakes -----------------------------------------------------------

def _round16_ties_away(v):
    a = abs(v)
    if a >= 65520:
        return np.copysign(np.inf, v)
    e = max(int(np.floor(np.log2(a))) if a > 0 else -14, -14)
    ulp = 2.0 ** (e - 10)
    return float(np.copysign(np.floor(a / ulp + 0.5) * ulp, v))


def _int8_scale_128(T):
    T = np.asarray(T, np.float64)
    s = np.max(np.abs(T)) / 128
    return (np.clip(np.rint(T / s), -127, 127) * s if s > 0 else T.copy()), s


def _int8_truncating(T):
    T = np.asarray(T, np.float64)
    s = np.max(np.abs(T)) / 127
    return (np.trunc(T / s) * s if s > 0 else T.copy()), s


@pytest.mark.parametrize("pin,broken", [(pin_fp16, _round16_ties_away), (pin_int8, _int8_scale_128),
                                        (pin_int8, _int8_truncating)],
                         ids=["fp16_ties_away", "int8_scale_128", "int8_truncating"])
def test_planted_quantisation_mistake_is_caught(pin, broken):
    with pytest.raises(AssertionError):
        pin(broken)

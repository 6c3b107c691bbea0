"""The library's host decomposition fitter (fluxbin_fit, fluxbin_fit_hybrid,
C++ with host threads) against the fp64 oracle restatement of the same steps
(oracle/fit.py): FluxBin summary, Section 3 "Parameter Optimization",
Appendix A.1 (closed-form scales), A.2 (joint sign search), Section 3
"Salient-Aware Hybrid Bases".

Both sides take every sign decision in fp64, so the signs must agree bit for
bit; scales and the objective agree to fp64 rounding (the two sum in
different orders).  Inputs: seeded dense matrices W_ij = a_i b_j z_ij with
a, b ~ LogNormal(0, 0.5) and z ~ N(0, 1) (the row and column anisotropy the
row-column decomposition targets) and seeded column weights in [0.2, 1.2).
"""
import ctypes

import numpy as np
import pytest

from lut_binary_basis_b200 import fluxbin
from oracle import fit as F

RTOL = 1e-10


def dense_w(seed, M, N):
    g = np.random.default_rng(seed)
    return (np.exp(0.5 * g.standard_normal(M))[:, None] * np.exp(0.5 * g.standard_normal(N))[None, :]
            * g.standard_normal((M, N)))


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


@pytest.mark.parametrize("M,N,nb,G,iters,weighted", [
    (64, 96, 1, 0, 3, False), (130, 257, 2, 0, 6, True), (100, 384, 2, 128, 5, True),
    (33, 200, 3, 64, 4, False), (70, 64, 4, 16, 3, True), (1, 1, 2, 0, 2, False), (50, 40, 2, 0, 0, True)])
def test_fit_matches_oracle(M, N, nb, G, iters, weighted):
    W = dense_w(M * 1000 + N, M, N)
    h = np.random.default_rng(N).random(N) + 0.2 if weighted else None
    s, r, c, obj = fluxbin.fluxbin_fit(W, nb, G, iters, h)
    s2, r2, c2, hist = F.fit(W, nb, G, iters, h, history=True)
    assert np.array_equal(s, s2)
    assert rel(r, np.stack(r2)) <= RTOL and rel(c, np.stack(c2)) <= RTOL
    assert abs(obj - hist[-1]) <= RTOL * hist[-1]


@pytest.mark.parametrize("G,Gs,weighted", [(0, 0, False), (128, 16, True), (64, 0, True)])
def test_fit_hybrid_matches_oracle(G, Gs, weighted):
    M, N = 90, 512
    W = dense_w(7 + G + Gs, M, N)
    S = np.sort(np.random.default_rng(3).choice(N, 48, replace=False)).astype(np.int32)
    h = np.random.default_rng(4).random(N) + 0.2 if weighted else None
    s, r, c, ss, rs, cs, obj = fluxbin.fluxbin_fit_hybrid(W, 2, S, 2, G, Gs, 4, h)
    (gs, gr, gc), (os_, or_, oc) = F.fit_hybrid(W, S, 2, 2, G, Gs, 4, h)
    assert np.array_equal(s, gs) and np.array_equal(ss, os_)
    for a, b in ((r, gr), (c, gc), (rs, or_), (cs, oc)):
        assert rel(a, np.stack(b)) <= RTOL
    full = F.reconstruct(gs, gr, gc, G)
    full[:, S] += F.reconstruct(os_, or_, oc, Gs)
    hh = np.ones(N) if h is None else h
    want = float(np.sum(hh[None, :] * (W - full) ** 2))
    assert abs(obj - want) <= RTOL * want


def test_fitted_layer_packs_and_round_trips_to_fp16():
    """The fitter's outputs are the arrays the packer takes: the fitted signs
    pack bit-exactly like any other, and the fp16-rounded scales form a layer
    whose reconstruction stays close to the fp64 fit."""
    from lut_binary_basis_b200.synth import LayerData, LayerSpec
    from oracle import layout
    M, N = 96, 256
    W = dense_w(11, M, N)
    S = np.sort(np.random.default_rng(12).choice(N, 32, replace=False)).astype(np.int32)
    s, r, c, ss, rs, cs, obj = fluxbin.fluxbin_fit_hybrid(W, 2, S, 1, 128, 0, 5)
    spec = LayerSpec("fit", M, N, 2, 1, 32, 8, row_scale_group=128)
    layer = LayerData(spec, s, r.astype(np.float16), c.astype(np.float16), S, ss, rs.astype(np.float16),
                      cs.astype(np.float16))
    words, swords = fluxbin.fluxbin_pack(fluxbin.LayerDesc.of(spec), layer.signs, layer.sal_signs, layer.sal_idx)
    assert np.array_equal(words, layout.pack_branch(s, 8))
    assert np.array_equal(swords, layout.pack_branch(ss, 8))
    full = F.reconstruct(s, list(r), list(c), 128)
    full[:, S] += F.reconstruct(ss, list(rs), list(cs), 0)
    full16 = F.reconstruct(s, list(layer.r.astype(np.float64)), list(layer.c.astype(np.float64)), 128)
    full16[:, S] += F.reconstruct(ss, list(layer.rs.astype(np.float64)), list(layer.cs.astype(np.float64)), 0)
    assert np.linalg.norm(full16 - full) <= 2e-3 * np.linalg.norm(full)
    assert np.sum((W - full) ** 2) == pytest.approx(obj, rel=1e-9)


def test_fit_argument_errors():
    L = fluxbin.lib()
    W = np.zeros((4, 4))
    p = W.ctypes.data_as(ctypes.c_void_p)
    out = np.zeros(64)
    q = out.ctypes.data_as(ctypes.c_void_p)
    assert L.fluxbin_fit(4, 4, 0, 0, 1, p, None, q, q, q, None) == -4
    assert L.fluxbin_fit(4, 4, 9, 0, 1, p, None, q, q, q, None) == -4
    assert L.fluxbin_fit(-1, 4, 1, 0, 1, p, None, q, q, q, None) == -2
    assert L.fluxbin_fit(4, 4, 1, 0, -1, p, None, q, q, q, None) == -2
    assert L.fluxbin_fit(4, 4, 1, 0, 1, None, None, q, q, q, None) == -1
    hbad = np.array([1.0, -1.0, 1.0, 1.0])
    assert L.fluxbin_fit(4, 4, 1, 0, 1, p, hbad.ctypes.data_as(ctypes.c_void_p), q, q, q, None) == -2
    idx = np.array([2, 1], np.int32)
    assert L.fluxbin_fit_hybrid(4, 4, 1, 0, 1, 2, idx.ctypes.data_as(ctypes.c_void_p), 0, 1, p, None, q, q, q,
                                q, q, q, None) == -2
    assert L.fluxbin_fit(0, 0, 1, 0, 1, None, None, None, None, None, None) == 0


@pytest.mark.gpu
def test_fitted_layer_runs_on_the_device():
    """A layer produced by the fitter (scales rounded to fp16, packed by the
    library) through fluxbin_linear matches the oracle on that layer, and its
    output approximates W x about as well as the fit approximates W."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    from lut_binary_basis_b200 import synth
    from lut_binary_basis_b200.synth import LayerData, LayerSpec
    from test_gpu_parity import assert_close, run_linear
    M, N = 1024, 2048
    W = dense_w(21, M, N)
    S = np.concatenate([blk * 128 + np.sort(np.random.default_rng(22 + blk).choice(128, 16, replace=False))
                        for blk in range(N // 128)]).astype(np.int32)
    s, r, c, ss, rs, cs, obj = fluxbin.fluxbin_fit_hybrid(W, 2, S, 2, 128, 16, 6)
    spec = LayerSpec("fit", M, N, 2, 2, S.size, 8, row_scale_group=128, sal_scale_group=16)
    layer = LayerData(spec, s, r.astype(np.float16), c.astype(np.float16), S, ss, rs.astype(np.float16),
                      cs.astype(np.float16))
    x = synth.make_x(spec, 2, [23])
    got = run_linear(layer, x)
    ref = oracle.linear(layer, x)
    assert_close(got, ref, layer, x)
    exact = x.astype(np.float64) @ W.T
    fit_rel = np.sqrt(obj / np.sum(W * W))
    out_rel = np.linalg.norm(got - exact) / np.linalg.norm(exact)
    assert out_rel <= 2 * fit_rel + 1e-2

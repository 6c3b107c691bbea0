"""FluxBin fp64 CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it, and it shares no code
with that path.

The arithmetic lives in ``fluxbin_oracle.c`` (plain C, fp64), compiled on
first use into ``liboracle.so`` next to it.  This module only marshals numpy
arrays: fp16 inputs are widened to fp64 with ``astype`` (exact).

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against
closed forms, invariants, library routines on special cases and brute force;
none of them is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fluxbin_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, OpenMP) into liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i64, i32 = ctypes.c_int64, ctypes.c_int
            lib.oracle_linear_rows.argtypes = [i64, i64, i32, i32, P, P, P, i32, i64, i32, P, P, P, P,
                                               i32, P, i64, P, P]
            lib.oracle_linear_rows.restype = None
            lib.oracle_lut_linear_rows.argtypes = [i64, i64, i32, i32, P, P, P, i32, i64, i32, P, P, P, P,
                                                   i32, i32, i32, i32, P, i64, P, P]
            lib.oracle_rmsnorm.argtypes = [i64, P, P, ctypes.c_double, P]
            lib.oracle_rmsnorm.restype = None
            lib.oracle_round_fp16.argtypes = [ctypes.c_double]
            lib.oracle_round_fp16.restype = ctypes.c_double
            lib.oracle_quantize_table_int8.argtypes = [P, i64]
            lib.oracle_quantize_table_int8.restype = ctypes.c_double
            lib.oracle_lut_linear_rows.restype = i32
            lib.oracle_lut_table.argtypes = [P, i32, P]
            lib.oracle_lut_table_sym.argtypes = [P, i32, P]
            lib.oracle_lut_lookup_sym.argtypes = [P, i32, i64]
            lib.oracle_lut_lookup_sym.restype = ctypes.c_double
            lib.oracle_rebuild_rows.argtypes = [i64, i64, i32, i32, P, P, P, i32, i64, i32, P, P, P, P, i64, P, P]
            lib.oracle_rebuild_rows.restype = None
            lib.oracle_gemv_rows.argtypes = [i64, i64, P, i32, P, P]
            lib.oracle_gemv_rows.restype = None
            lib.oracle_num_threads.restype = i32
            lib.oracle_set_num_threads.argtypes = [i32]
            _lib = lib
    return _lib


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a).astype(np.float64))


def _i8(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int8))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _unpack(layer):
    spec = layer.spec
    Ks = layer.sal_signs.shape[0] if layer.sal_signs.size else 0
    n_sal = int(layer.sal_idx.size)
    return dict(M=spec.M, N=spec.N, Kb=layer.signs.shape[0], G=spec.row_scale_group,
                signs=_i8(layer.signs), r=_f64(layer.r), c=_f64(layer.c),
                Ks=Ks if n_sal else 0, n_sal=n_sal, Gs=spec.sal_scale_group,
                sal_signs=_i8(layer.sal_signs), rs=_f64(layer.rs), cs=_f64(layer.cs),
                sal_idx=np.ascontiguousarray(layer.sal_idx, dtype=np.int32))


def _rows(M: int, rows: Optional[Sequence[int]]) -> np.ndarray:
    if rows is None:
        return np.arange(M, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64))


def linear(layer, x, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """y[b][q] = (W x[b])[rows[q]] by the definition (W rebuilt row by row in fp64).

    ``layer`` carries ``spec`` (M, N, row_scale_group, sal_scale_group) and the
    arrays signs, r, c, sal_idx, sal_signs, rs, cs in the documented layouts;
    ``x`` is [B][N].  Returns float64 [B][len(rows)].
    """
    L = _unpack(layer)
    xx = _f64(x)
    B = xx.shape[0]
    rr = _rows(L["M"], rows)
    y = np.zeros((B, rr.size), np.float64)
    if rr.size == 0 or B == 0:
        return y
    assert xx.shape[1] == L["N"]
    _load().oracle_linear_rows(L["M"], L["N"], L["Kb"], L["G"], _ptr(L["signs"]), _ptr(L["r"]), _ptr(L["c"]),
                               L["Ks"], L["n_sal"], L["Gs"], _ptr(L["sal_signs"]), _ptr(L["rs"]), _ptr(L["cs"]),
                               _ptr(L["sal_idx"]), B, _ptr(xx), rr.size, _ptr(rr), _ptr(y))
    return y


def rebuild_rows(layer, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Rows of W = sum_k diag(r_k) B_k diag(c_k) (+ the salient branch at its
    true columns), rebuilt in fp64: float64 [len(rows)][N]."""
    L = _unpack(layer)
    rr = _rows(L["M"], rows)
    W = np.zeros((rr.size, L["N"]), np.float64)
    if rr.size == 0 or L["N"] == 0:
        return W
    _load().oracle_rebuild_rows(L["M"], L["N"], L["Kb"], L["G"], _ptr(L["signs"]), _ptr(L["r"]), _ptr(L["c"]),
                                L["Ks"], L["n_sal"], L["Gs"], _ptr(L["sal_signs"]), _ptr(L["rs"]), _ptr(L["cs"]),
                                _ptr(L["sal_idx"]), rr.size, _ptr(rr), _ptr(W))
    return W


def gemv_rows(W: np.ndarray, x) -> np.ndarray:
    """y[b][q] = W[q] . x[b] in fp64 for rows already rebuilt by rebuild_rows."""
    W = np.ascontiguousarray(W, dtype=np.float64)
    xx = _f64(x)
    y = np.zeros((xx.shape[0], W.shape[0]), np.float64)
    if W.size == 0 or xx.shape[0] == 0:
        return y
    assert xx.shape[1] == W.shape[1]
    _load().oracle_gemv_rows(W.shape[1], W.shape[0], _ptr(W), xx.shape[0], _ptr(xx), _ptr(y))
    return y


TABLE_QUANT = {"none": 0, "fp16": 1, "int8": 2}


def rmsnorm(h, gamma, eps: float) -> np.ndarray:
    """x = h * gamma / sqrt(mean(h^2) + eps) in fp64: the element-wise
    operator taken to precede a layer whose table precompute is fused into it
    (one activation row, [N])."""
    hh = _f64(np.asarray(h).reshape(-1)).copy()
    gg = _f64(np.asarray(gamma).reshape(-1)).copy()
    assert hh.size == gg.size and hh.size > 0
    x = np.zeros(hh.size, np.float64)
    _load().oracle_rmsnorm(hh.size, _ptr(hh), _ptr(gg), float(eps), _ptr(x))
    return x


def linear_rmsnorm(layer, h, gamma, eps: float) -> np.ndarray:
    """y = W rmsnorm(h) for one activation row, [1][M]."""
    return linear(layer, rmsnorm(h, gamma, eps)[None, :])


def round_fp16(v: float) -> float:
    """The binary16 value nearest to v (ties to even)."""
    return float(_load().oracle_round_fp16(float(v)))


def quantize_table_int8(T) -> tuple:
    """INT8 quantisation of one table with one scale: returns (entries, scale)."""
    tt = _f64(T).copy()
    s = float(_load().oracle_quantize_table_int8(_ptr(tt), tt.size))
    return tt, s


def lut_linear(layer, x, mu: int, sym: bool = False, rows: Optional[Sequence[int]] = None,
               tables: str = "none") -> np.ndarray:
    """The same layer evaluated by the method's steps: scale-fused tables of
    2^mu signed partial sums per sub-vector, looked up by the sign patterns
    (``sym``: symmetric half tables; ``tables``: table quantisation, "none",
    "fp16" or "int8" with one scale per table)."""
    L = _unpack(layer)
    xx = _f64(x)
    B = xx.shape[0]
    rr = _rows(L["M"], rows)
    y = np.zeros((B, rr.size), np.float64)
    if rr.size == 0 or B == 0:
        return y
    rc = _load().oracle_lut_linear_rows(L["M"], L["N"], L["Kb"], L["G"], _ptr(L["signs"]), _ptr(L["r"]),
                                        _ptr(L["c"]), L["Ks"], L["n_sal"], L["Gs"], _ptr(L["sal_signs"]),
                                        _ptr(L["rs"]), _ptr(L["cs"]), _ptr(L["sal_idx"]), int(mu), int(bool(sym)),
                                        TABLE_QUANT[tables], B, _ptr(xx), rr.size, _ptr(rr), _ptr(y))
    if rc != 0:
        raise ValueError("scale block sizes must be multiples of mu")
    return y


def lut_table(v, mu: int) -> np.ndarray:
    vv = _f64(v)
    assert vv.size == mu
    T = np.zeros(1 << mu, np.float64)
    _load().oracle_lut_table(_ptr(vv), mu, _ptr(T))
    return T


def lut_table_sym(v, mu: int) -> np.ndarray:
    vv = _f64(v)
    assert vv.size == mu
    T = np.zeros(1 << (mu - 1), np.float64)
    _load().oracle_lut_table_sym(_ptr(vv), mu, _ptr(T))
    return T


def lut_lookup_sym(Th, mu: int, p: int) -> float:
    tt = _f64(Th)
    return float(_load().oracle_lut_lookup_sym(_ptr(tt), mu, int(p)))

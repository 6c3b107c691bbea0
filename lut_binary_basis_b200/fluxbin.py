"""ctypes binding of libfluxbin.so (include/fluxbin.h), argument marshalling only.

Every computation runs in the library's CUDA kernels; this module converts
torch tensors and numpy arrays to pointers, sizes and the current CUDA stream,
and raises ``FluxbinError`` on a non-zero status.  There is no fallback: if
the shared library is missing, the first call raises ``FluxbinLibraryMissing``.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import threading
from typing import Optional, Tuple

import numpy as np

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfluxbin.so")

FLAG_ACCUMULATE = 1
FLAG_Y_FP32 = 2
FLAG_EARLY_WEIGHTS = 4
FLAG_PATH_LUT = 8
FLAG_PATH_TC = 16
FLAG_TEST_WAIT_TIMEOUT = 32
FLAG_SEPARATE_TABLES = 64

STATUS = {0: "FLUXBIN_OK", -1: "FLUXBIN_ERR_INVALID_ARG", -2: "FLUXBIN_ERR_BAD_SHAPE",
          -3: "FLUXBIN_ERR_MISALIGNED", -4: "FLUXBIN_ERR_UNSUPPORTED", -5: "FLUXBIN_ERR_SMEM_BUDGET",
          -6: "FLUXBIN_ERR_WORKSPACE", -7: "FLUXBIN_ERR_CUDA", -8: "FLUXBIN_ERR_SCRATCH_LIMIT"}

STATIC_SCRATCH_BYTES = 4 << 20


class FluxbinLibraryMissing(ImportError):
    pass


class FluxbinError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = f"; {fluxbin_last_error()}" if status == -7 else ""
        super().__init__(f"{where}: {STATUS.get(status, status)} ({fluxbin_status_string(status)}{detail})")


class LayerDesc(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int32), ("N", ctypes.c_int32), ("Kb", ctypes.c_int32), ("Ks", ctypes.c_int32),
                ("n_sal", ctypes.c_int32), ("mu", ctypes.c_int32), ("row_scale_group", ctypes.c_int32),
                ("sal_scale_group", ctypes.c_int32)]

    @classmethod
    def of(cls, spec) -> "LayerDesc":
        Ks = spec.Ks if (spec.Ks and spec.n_sal) else 0
        return cls(spec.M, spec.N, spec.Kb, Ks, spec.n_sal if Ks else 0, spec.mu, spec.row_scale_group,
                   spec.sal_scale_group if Ks else 0)


_lock = threading.Lock()
_lib = None


def lib():
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise FluxbinLibraryMissing(f"{LIB_PATH} is not built (run __graft_entry__.build())")
            L = ctypes.CDLL(LIB_PATH)
            P, i32, u32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32, ctypes.c_size_t
            L.fluxbin_status_string.argtypes = [ctypes.c_int]
            L.fluxbin_status_string.restype = ctypes.c_char_p
            L.fluxbin_version.restype = ctypes.c_int
            L.fluxbin_last_error.restype = ctypes.c_char_p
            L.fluxbin_packed_sizes.argtypes = [P, ctypes.POINTER(sz), ctypes.POINTER(sz)]
            L.fluxbin_pack.argtypes = [P, P, P, P, P, P]
            L.fluxbin_workspace_bytes.argtypes = [i32, i32, ctypes.POINTER(sz)]
            L.fluxbin_layer_workspace_bytes.argtypes = [P, i32, ctypes.POINTER(sz)]
            L.fluxbin_lut_gemv.argtypes = [i32, i32, i32, i32, i32, i32, P, P, P, P, P, i32, P, u32, P, sz, P]
            L.fluxbin_linear.argtypes = [P, P, P, P, P, P, P, P, P, i32, P, u32, P, sz, P]
            L.fluxbin_linear_static_scratch.argtypes = [P, P, P, P, P, P, P, P, P, i32, P, u32, P]
            L.fluxbin_linear_rmsnorm.argtypes = [P, P, P, P, P, P, P, P, P, P, ctypes.c_float, P, P, u32, P, sz, P]
            L.fluxbin_device_status.argtypes = [ctypes.POINTER(u32)]
            L.fluxbin_fit.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P, P]
            L.fluxbin_fit_hybrid.argtypes = [i32, i32, i32, i32, i32, i32, P, i32, i32, P, P, P, P, P, P, P, P, P]
            for f in ("fluxbin_packed_sizes", "fluxbin_pack", "fluxbin_workspace_bytes",
                      "fluxbin_layer_workspace_bytes", "fluxbin_lut_gemv",
                      "fluxbin_linear", "fluxbin_linear_static_scratch", "fluxbin_linear_rmsnorm",
                      "fluxbin_device_status", "fluxbin_fit",
                      "fluxbin_fit_hybrid"):
                getattr(L, f).restype = ctypes.c_int
            _lib = L
    return _lib


def _check(st: int, where: str) -> None:
    if st != 0:
        raise FluxbinError(st, where)


def fluxbin_status_string(status: int) -> str:
    return lib().fluxbin_status_string(int(status)).decode()


def fluxbin_last_error() -> str:
    return lib().fluxbin_last_error().decode()


def fluxbin_device_status() -> int:
    """Device-side status flags of the current device (read and cleared)."""
    v = ctypes.c_uint32(0)
    _check(lib().fluxbin_device_status(ctypes.byref(v)), "fluxbin_device_status")
    return int(v.value)


def fluxbin_version() -> int:
    return lib().fluxbin_version()


def fluxbin_packed_sizes(desc: LayerDesc) -> Tuple[int, int]:
    wb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().fluxbin_packed_sizes(ctypes.byref(desc), ctypes.byref(wb), ctypes.byref(sb)),
           "fluxbin_packed_sizes")
    return wb.value, sb.value


def _np_ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def fluxbin_pack(desc: LayerDesc, signs: np.ndarray, sal_signs: Optional[np.ndarray] = None,
                 sal_idx: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Host packer: int8 +-1 signs -> uint32 words (global, salient)."""
    wb, sb = fluxbin_packed_sizes(desc)
    words = np.zeros(wb // 4, np.uint32)
    swords = np.zeros(sb // 4, np.uint32)
    s = np.ascontiguousarray(signs, dtype=np.int8)
    ss = np.ascontiguousarray(sal_signs, dtype=np.int8) if sal_signs is not None else None
    si = np.ascontiguousarray(sal_idx, dtype=np.int32) if sal_idx is not None else None
    _check(lib().fluxbin_pack(ctypes.byref(desc), _np_ptr(s), _np_ptr(ss), _np_ptr(si), _np_ptr(words),
                              _np_ptr(swords) if sb else None), "fluxbin_pack")
    return words, swords


def fluxbin_workspace_bytes(M: int, B: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().fluxbin_workspace_bytes(int(M), int(B), ctypes.byref(n)), "fluxbin_workspace_bytes")
    return n.value


def fluxbin_layer_workspace_bytes(desc: LayerDesc, B: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().fluxbin_layer_workspace_bytes(ctypes.byref(desc), int(B), ctypes.byref(n)),
           "fluxbin_layer_workspace_bytes")
    return n.value


def _dptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def fluxbin_lut_gemv(M: int, N: int, ncols: int, nbases: int, mu: int, row_scale_group: int, words, r, c, gather,
                     x, B: int, y, flags: int = FLAG_Y_FP32, workspace=None, workspace_bytes: Optional[int] = None,
                     stream=None) -> None:
    wsb = workspace_bytes if workspace_bytes is not None else (
        workspace.numel() * workspace.element_size() if workspace is not None else 0)
    _check(lib().fluxbin_lut_gemv(M, N, ncols, nbases, mu, row_scale_group, _dptr(words), _dptr(r), _dptr(c),
                                  _dptr(gather), _dptr(x), B, _dptr(y), flags, _dptr(workspace), wsb,
                                  _stream(stream)), "fluxbin_lut_gemv")


def fluxbin_linear(desc: LayerDesc, words, r, c, swords, rs, cs, idx, x, B: int, y, flags: int = FLAG_Y_FP32,
                   workspace=None, workspace_bytes: Optional[int] = None, stream=None) -> None:
    wsb = workspace_bytes if workspace_bytes is not None else (
        workspace.numel() * workspace.element_size() if workspace is not None else 0)
    _check(lib().fluxbin_linear(ctypes.byref(desc), _dptr(words), _dptr(r), _dptr(c), _dptr(swords), _dptr(rs),
                                _dptr(cs), _dptr(idx), _dptr(x), B, _dptr(y), flags, _dptr(workspace), wsb,
                                _stream(stream)), "fluxbin_linear")


def fluxbin_linear_rmsnorm(desc: LayerDesc, words, r, c, swords, rs, cs, idx, h, gamma, eps: float, x_out, y,
                           flags: int = FLAG_Y_FP32, workspace=None, workspace_bytes: Optional[int] = None,
                           stream=None) -> None:
    """y (+)= W (h * gamma / sqrt(mean(h^2) + eps)) at batch 1, the table
    precompute fused with the RMS normalisation (include/fluxbin.h);
    x_out (fp16 [N] or None) receives the normalised activation."""
    wsb = workspace_bytes if workspace_bytes is not None else (
        workspace.numel() * workspace.element_size() if workspace is not None else 0)
    _check(lib().fluxbin_linear_rmsnorm(ctypes.byref(desc), _dptr(words), _dptr(r), _dptr(c), _dptr(swords),
                                        _dptr(rs), _dptr(cs), _dptr(idx), _dptr(h), _dptr(gamma), float(eps),
                                        _dptr(x_out), _dptr(y), flags, _dptr(workspace), wsb, _stream(stream)),
           "fluxbin_linear_rmsnorm")


def fluxbin_linear_static_scratch(desc: LayerDesc, words, r, c, swords, rs, cs, idx, x, B: int, y,
                                  flags: int = FLAG_Y_FP32, stream=None) -> None:
    """fluxbin_linear without a workspace argument, for callers that cannot
    allocate device memory: the split-K scratch is the library's own fixed
    device array (STATIC_SCRATCH_BYTES per device).  Calls that may overlap on
    the GPU share that array and must be ordered on one stream."""
    _check(lib().fluxbin_linear_static_scratch(ctypes.byref(desc), _dptr(words), _dptr(r), _dptr(c), _dptr(swords),
                                               _dptr(rs), _dptr(cs), _dptr(idx), _dptr(x), B, _dptr(y), flags,
                                               _stream(stream)), "fluxbin_linear_static_scratch")


def _scale_shape(nb: int, M: int, ncols: int, G: int):
    return (nb, -(-ncols // G), M) if G > 0 else (nb, M)


def fluxbin_fit(W: np.ndarray, nbases: int, row_scale_group: int = 0, iters: int = 10,
                col_weight: Optional[np.ndarray] = None):
    """Host decomposition fitting of one branch (include/fluxbin.h): returns
    (signs int8 [nb][M][N], r fp64, c fp64 [nb][N], objective)."""
    W = np.ascontiguousarray(W, dtype=np.float64)
    M, N = W.shape
    h = None if col_weight is None else np.ascontiguousarray(col_weight, dtype=np.float64)
    signs = np.zeros((nbases, M, N), np.int8)
    r = np.zeros(_scale_shape(nbases, M, N, row_scale_group), np.float64)
    c = np.zeros((nbases, N), np.float64)
    obj = ctypes.c_double()
    _check(lib().fluxbin_fit(M, N, nbases, row_scale_group, iters, _np_ptr(W), _np_ptr(h), _np_ptr(signs),
                             _np_ptr(r), _np_ptr(c), ctypes.byref(obj)), "fluxbin_fit")
    return signs, r, c, obj.value


def fluxbin_fit_hybrid(W: np.ndarray, Kb: int, sal_idx: np.ndarray, Ks: int, row_scale_group: int = 0,
                       sal_scale_group: int = 0, iters: int = 10, col_weight: Optional[np.ndarray] = None):
    """Global bases, then the salient refinement on the residual at columns
    sal_idx: returns (signs, r, c, sal_signs, rs, cs, objective)."""
    W = np.ascontiguousarray(W, dtype=np.float64)
    M, N = W.shape
    idx = np.ascontiguousarray(sal_idx, dtype=np.int32)
    ns = int(idx.size) if Ks else 0
    h = None if col_weight is None else np.ascontiguousarray(col_weight, dtype=np.float64)
    signs = np.zeros((Kb, M, N), np.int8)
    r = np.zeros(_scale_shape(Kb, M, N, row_scale_group), np.float64)
    c = np.zeros((Kb, N), np.float64)
    ss = np.zeros((Ks, M, ns), np.int8)
    rs = np.zeros(_scale_shape(Ks, M, ns, sal_scale_group), np.float64)
    cs = np.zeros((Ks, ns), np.float64)
    obj = ctypes.c_double()
    _check(lib().fluxbin_fit_hybrid(M, N, Kb, row_scale_group, Ks, ns, _np_ptr(idx), sal_scale_group, iters,
                                    _np_ptr(W), _np_ptr(h), _np_ptr(signs), _np_ptr(r), _np_ptr(c), _np_ptr(ss),
                                    _np_ptr(rs), _np_ptr(cs), ctypes.byref(obj)), "fluxbin_fit_hybrid")
    return signs, r, c, ss, rs, cs, obj.value


def pack_host(layer) -> dict:
    """Pack a host layer (``LayerData``) with the library's packer: the host
    arrays a device layer is made of (no CUDA involved)."""
    desc = LayerDesc.of(layer.spec)
    words, swords = fluxbin_pack(desc, layer.signs, layer.sal_signs if desc.Ks else None,
                                 layer.sal_idx if desc.Ks else None)
    return {"desc": desc, "words": words, "r": layer.r, "c": layer.c, "swords": swords, "rs": layer.rs,
            "cs": layer.cs, "idx": layer.sal_idx.astype(np.int32)}


@dataclasses.dataclass
class DeviceLayer:
    """One packed layer resident on a CUDA device (torch owns the memory)."""

    desc: LayerDesc
    words: "object"
    r: "object"
    c: "object"
    swords: "object"
    rs: "object"
    cs: "object"
    idx: "object"

    @classmethod
    def from_host(cls, layer, device="cuda") -> "DeviceLayer":
        """Pack a host layer (``LayerData``) with the library's packer and copy it to ``device``."""
        return cls.from_packed(pack_host(layer), device)

    @classmethod
    def from_packed(cls, packed: dict, device="cuda") -> "DeviceLayer":
        """Copy the arrays of ``pack_host`` to ``device``."""
        import torch

        def dev(a, dtype):
            a = np.ascontiguousarray(a)
            t = torch.from_numpy(a.view(dtype) if a.size else np.zeros(1, dtype))
            return t.to(device)

        p = packed
        return cls(p["desc"], dev(p["words"], np.int32), dev(p["r"], np.float16), dev(p["c"], np.float16),
                   dev(p["swords"], np.int32), dev(p["rs"], np.float16), dev(p["cs"], np.float16),
                   dev(p["idx"], np.int32))

    def workspace(self, B: int, device=None):
        """A zero-filled workspace of fluxbin_layer_workspace_bytes(desc, B) bytes
        (room for the batch-1 table buffer where the layer can use one)."""
        import torch
        n = max(fluxbin_layer_workspace_bytes(self.desc, B), 256)
        return torch.zeros(n // 4, dtype=torch.int32, device=device if device is not None else self.words.device)

    def linear(self, x, y, flags: int = FLAG_Y_FP32, workspace=None, stream=None) -> None:
        B = x.shape[0] if x.dim() == 2 else 1
        fluxbin_linear(self.desc, self.words, self.r, self.c, self.swords, self.rs, self.cs, self.idx, x, B, y,
                       flags, workspace, None, stream)

    def linear_rmsnorm(self, h, gamma, eps: float, y, flags: int = FLAG_Y_FP32, workspace=None, x_out=None,
                       stream=None) -> None:
        fluxbin_linear_rmsnorm(self.desc, self.words, self.r, self.c, self.swords, self.rs, self.cs, self.idx, h,
                               gamma, eps, x_out, y, flags, workspace, None, stream)


def new_workspace(M: int, B: int, device="cuda"):
    """A zero-filled workspace of fluxbin_workspace_bytes(M, B) bytes (at least 256)."""
    import torch
    n = max(fluxbin_workspace_bytes(M, B), 256)
    return torch.zeros(n // 4, dtype=torch.int32, device=device)

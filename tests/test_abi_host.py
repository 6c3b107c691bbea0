"""Host-side checks of libfluxbin.so (no GPU needed): the library loads and
exports every entry point include/fluxbin.h declares, the host packer is
bit-exact against the independent naive packer, and argument errors come
back as status codes before any CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

from lut_binary_basis_b200 import fluxbin
from lut_binary_basis_b200.fluxbin import LayerDesc
from lut_binary_basis_b200.synth import LayerSpec, make_layer
from oracle import layout

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fluxbin.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(fluxbin_\w+)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert {"fluxbin_pack", "fluxbin_lut_gemv", "fluxbin_linear", "fluxbin_status_string"} <= set(names)
    L = ctypes.CDLL(fluxbin.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version():
    assert fluxbin.fluxbin_status_string(0) == "ok"
    for code in range(-7, 0):
        assert fluxbin.fluxbin_status_string(code) not in ("", "unknown status")
    assert fluxbin.fluxbin_status_string(-99) == "unknown status"
    assert fluxbin.fluxbin_version() >= 10000


def _signs(rng, shape):
    return (rng.integers(0, 2, size=shape) * 2 - 1).astype(np.int8)


@pytest.mark.parametrize("M,N,Kb,Ks,n_sal,mu", [
    (64, 256, 1, 0, 0, 4), (33, 300, 2, 1, 17, 8), (100, 1000, 4, 2, 40, 8), (1, 8, 2, 4, 3, 4),
    (257, 129, 2, 1, 5, 4), (32, 4096, 2, 1, 205, 8)])
def test_pack_bit_exact_against_naive_packer(M, N, Kb, Ks, n_sal, mu):
    rng = np.random.default_rng(M + N)
    spec = LayerSpec("p", M, N, Kb, Ks, n_sal, mu)
    d = make_layer(spec, [M, N, Kb])
    desc = LayerDesc.of(spec)
    words, swords = fluxbin.fluxbin_pack(desc, d.signs, d.sal_signs if Ks else None, d.sal_idx if Ks else None)
    ref = layout.pack_branch(d.signs, mu)
    assert words.dtype == np.uint32 and np.array_equal(words, ref)
    if Ks:
        assert np.array_equal(swords, layout.pack_branch(d.sal_signs, mu))
        assert np.array_equal(layout.unpack_branch(swords, M, n_sal, Ks, mu), d.sal_signs)
    assert np.array_equal(layout.unpack_branch(words, M, N, Kb, mu), d.signs)
    wb, sb = fluxbin.fluxbin_packed_sizes(desc)
    assert wb == 4 * layout.branch_words(M, N, Kb, mu)
    assert sb == (4 * layout.branch_words(M, n_sal, Ks, mu) if Ks else 0)
    del rng


@pytest.mark.parametrize("M,N,Kb,Ks,n_sal,mu,Gs,gsv", [
    (70, 512, 2, 2, 64, 8, 16, 2), (33, 300, 1, 1, 100, 8, 8, 1), (64, 1024, 2, 4, 96, 8, 32, 4),
    (40, 256, 2, 2, 64, 4, 8, 2), (50, 512, 4, 1, 60, 4, 16, 4), (32, 4096, 2, 2, 512, 8, 16, 2)])
def test_pack_grouped_salient_bit_exact(M, N, Kb, Ks, n_sal, mu, Gs, gsv):
    """Salient row scales finer than a unit use the grouped visit order."""
    spec = LayerSpec("g", M, N, Kb, Ks, n_sal, mu, sal_scale_group=Gs)
    d = make_layer(spec, [M, N, Gs])
    desc = LayerDesc.of(spec)
    words, swords = fluxbin.fluxbin_pack(desc, d.signs, d.sal_signs, d.sal_idx)
    assert np.array_equal(words, layout.pack_branch(d.signs, mu))
    assert np.array_equal(swords, layout.pack_branch(d.sal_signs, mu, gsv))
    assert np.array_equal(layout.unpack_branch(swords, M, n_sal, Ks, mu, gsv), d.sal_signs)
    # a different permutation of the same bits, except for one base with one
    # sub-vector per group, where both orders are the plain diagonal
    same = np.array_equal(swords, layout.pack_branch(d.sal_signs, mu))
    assert same == (Ks == 1 and gsv == 1)


def test_pack_rejects_bad_inputs():
    spec = LayerSpec("p", 8, 64, 1, 1, 4, 8)
    d = make_layer(spec, [1])
    desc = LayerDesc.of(spec)
    bad = d.signs.copy()
    bad[0, 3, 5] = 0
    with pytest.raises(fluxbin.FluxbinError) as e:
        fluxbin.fluxbin_pack(desc, bad, d.sal_signs, d.sal_idx)
    assert e.value.status == -2
    for idx in (np.array([3, 3, 7, 9]), np.array([5, 2, 7, 9]), np.array([1, 2, 3, 64]), np.array([-1, 2, 3, 4])):
        with pytest.raises(fluxbin.FluxbinError) as e:
            fluxbin.fluxbin_pack(desc, d.signs, d.sal_signs, idx.astype(np.int32))
        assert e.value.status == -2


@pytest.mark.parametrize("field,value,status", [
    ("mu", 5, -4), ("mu", 16, -4), ("Kb", 3, -4), ("Kb", 0, -4), ("Ks", 3, -4), ("M", -1, -2),
    ("n_sal", 70, -2), ("row_scale_group", 100, -4), ("row_scale_group", -2, -2),
    ("sal_scale_group", 12, -4), ("sal_scale_group", 24, -4), ("sal_scale_group", 64, -4)])
def test_desc_validation(field, value, status):
    desc = LayerDesc(32, 64, 2, 1, 4, 8, 0, 0)
    setattr(desc, field, value)
    with pytest.raises(fluxbin.FluxbinError) as e:
        fluxbin.fluxbin_packed_sizes(desc)
    assert e.value.status == status


def test_workspace_bytes():
    assert fluxbin.fluxbin_workspace_bytes(0, 4) == 0
    assert fluxbin.fluxbin_workspace_bytes(4096, 0) == 0
    n = fluxbin.fluxbin_workspace_bytes(4096, 1)
    assert n >= 4096 * 4 and n % 256 == 0
    assert fluxbin.fluxbin_workspace_bytes(4097, 3) >= 3 * 4128 * 4
    with pytest.raises(fluxbin.FluxbinError):
        fluxbin.fluxbin_workspace_bytes(-1, 1)


def _linear_status(desc, B=1, y=0x1000, flags=fluxbin.FLAG_Y_FP32, words=0x1000, x=0x2000):
    L = fluxbin.lib()
    return L.fluxbin_linear(ctypes.byref(desc), words, 0x3000, 0x4000, 0x5000, 0x6000, 0x7000, 0x8000, x, B, y,
                            flags, None, 0, None)


def test_device_entry_points_validate_before_any_cuda_call():
    desc = LayerDesc(32, 64, 2, 1, 4, 8, 0, 0)
    assert _linear_status(desc, B=0) == 0            # nothing to do
    assert _linear_status(LayerDesc(0, 64, 2, 1, 4, 8, 0, 0)) == 0
    assert _linear_status(desc, B=17) == -4
    assert _linear_status(desc, B=-1) == -2
    assert _linear_status(desc, y=0) == -1
    assert _linear_status(desc, y=0x1002) == -3      # fp32 y needs 4-byte alignment
    assert _linear_status(desc, words=0x1008) == -3  # packed words need 16-byte alignment
    assert _linear_status(desc, flags=128) == -1      # unknown flag
    assert _linear_status(desc, flags=fluxbin.FLAG_Y_FP32 | fluxbin.FLAG_SEPARATE_TABLES) == -6  # no table buffer
    assert _linear_status(LayerDesc(32, 64, 2, 1, 4, 6, 0, 0)) == -4
    L = fluxbin.lib()
    assert L.fluxbin_lut_gemv(32, 64, 65, 2, 8, 0, 0x1000, 0x2000, 0x3000, None, 0x4000, 1, 0x5000,
                              fluxbin.FLAG_Y_FP32, None, 0, None) == -2   # ncols > N without a gather
    assert L.fluxbin_lut_gemv(32, 64, 64, 3, 8, 0, 0x1000, 0x2000, 0x3000, None, 0x4000, 1, 0x5000,
                              fluxbin.FLAG_Y_FP32, None, 0, None) == -4
    assert L.fluxbin_linear(None, 0, 0, 0, 0, 0, 0, 0, 0, 1, 0, 0, None, 0, None) == -1


def test_layer_workspace_bytes():
    """Batch-1 mu = 8 layers with per-row scales add a table buffer of 64 KiB
    per pair of units (a unit is (32/nb)*mu columns of a branch); other layers
    and batch sizes need exactly fluxbin_workspace_bytes."""
    d = LayerDesc(28672, 8192, 2, 2, 246, 8, 0, 0)
    units = -(-8192 // 128) + -(-246 // 128)
    assert fluxbin.fluxbin_layer_workspace_bytes(d, 1) == \
        fluxbin.fluxbin_workspace_bytes(28672, 1) + -(-units // 2) * 65536
    for desc, B in ((d, 2), (LayerDesc(4096, 4096, 2, 1, 205, 4, 0, 0), 1),
                    (LayerDesc(4096, 4096, 2, 2, 512, 8, 128, 16), 1)):
        assert fluxbin.fluxbin_layer_workspace_bytes(desc, B) == fluxbin.fluxbin_workspace_bytes(desc.M, B)
    with pytest.raises(fluxbin.FluxbinError):
        fluxbin.fluxbin_layer_workspace_bytes(LayerDesc(4, 4, 3, 0, 0, 8, 0, 0), 1)

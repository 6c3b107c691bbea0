"""The entry point for callers that cannot allocate device memory.

Some callers have no way to hand the library a workspace: a plugin inside a
host program that owns all device memory through its own pool and forbids
direct cudaMalloc, or a latency-critical loop that must never call
cudaMalloc / cudaFree because they synchronise the device.
fluxbin_linear_static_scratch serves them with a fixed scratch array inside
the library.  This test calls it through the C-ABI, twice in a row, and
checks each result against the fp64 oracle and against fluxbin_linear given a
caller-allocated workspace, on launch plans that reduce inside a cluster, not
at all, through the scratch (LUT path) and on the tensor cores (whose split
items reduce through the scratch too).

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from lut_binary_basis_b200 import fluxbin, synth  # noqa: E402
from lut_binary_basis_b200.synth import LayerSpec  # noqa: E402

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3
ABS_FACTOR = 1e-2


def close(got, ref, layer, x):
    xn = np.linalg.norm(x.astype(np.float64), axis=1)
    mr = max(np.abs(layer.r.astype(np.float64)).max(initial=0), np.abs(layer.rs.astype(np.float64)).max(initial=0))
    mc = max(np.abs(layer.c.astype(np.float64)).max(initial=0), np.abs(layer.cs.astype(np.float64)).max(initial=0))
    for b in range(ref.shape[0]):
        assert np.linalg.norm(got[b] - ref[b]) <= REL_L2 * np.linalg.norm(ref[b])
        assert np.max(np.abs(got[b] - ref[b])) <= ABS_FACTOR * xn[b] * mr * mc


@pytest.mark.parametrize("sp,B", [
    (synth.layer_7b_proj(), 1),
    (LayerSpec("ragged", 2100, 777, 2, 1, 40, 8), 3),
    (LayerSpec("mu4", 1500, 1030, 2, 2, 60, 4), 5),
    (LayerSpec("wide", 256, 65536, 2, 1, 300, 8), 2),   # reduction through the scratch
    (LayerSpec("tc", 8192, 4096, 2, 1, 205, 8), 16),    # tensor cores, items reduced through the scratch
])
def test_static_scratch_matches_workspace_entry_point(sp, B):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    layer = synth.make_layer(sp, [123, sp.M, B])
    x = synth.make_x(sp, B, [124, sp.M, B])
    d = fluxbin.DeviceLayer.from_host(layer)
    xd = torch.from_numpy(x).cuda()
    y_ref = torch.zeros((B, sp.M), dtype=torch.float32, device="cuda")
    ws = fluxbin.new_workspace(sp.M, B)
    d.linear(xd, y_ref, fluxbin.FLAG_Y_FP32, ws)
    torch.cuda.synchronize()
    ref = y_ref.cpu().numpy().astype(np.float64)
    exact = oracle.linear(layer, x)
    close(ref, exact, layer, x)
    for call in range(2):
        y = torch.full((B, sp.M), float("nan"), dtype=torch.float32, device="cuda")
        fluxbin.fluxbin_linear_static_scratch(d.desc, d.words, d.r, d.c, d.swords, d.rs, d.cs, d.idx, xd, B, y,
                                              fluxbin.FLAG_Y_FP32)
        torch.cuda.synchronize()
        got = y.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)), f"call {call}"
        close(got, exact, layer, x)
        close(got, ref, layer, x)


def test_static_scratch_rejects_layers_beyond_its_size():
    # 300000 rows at batch 16 need more than the fixed scratch; rejected before any launch
    desc = fluxbin.LayerDesc(300000, 64, 2, 0, 0, 8, 0, 0)
    assert fluxbin.fluxbin_workspace_bytes(300000, 16) > fluxbin.STATIC_SCRATCH_BYTES
    L = fluxbin.lib()
    st = L.fluxbin_linear_static_scratch(ctypes.byref(desc), 0x1000, 0x2000, 0x3000, 0, 0, 0, 0, 0x4000, 16, 0x5000,
                                         fluxbin.FLAG_Y_FP32, None)
    assert st == -8


@pytest.mark.parametrize("sp,B", [
    (LayerSpec("large_b1", 16400, 8192, 2, 2, 246, 8), 1),   # warp-specialised batch-1 kernel
    (LayerSpec("pairs", 5000, 4096, 2, 1, 205, 8), 6),       # batch pairs on fp16-pair tables
])
def test_static_scratch_on_the_new_kernels(sp, B):
    """The static scratch behind the batch-1 and batch-pair kernels, whose
    plans split one CTA per SM through the scratch: two calls in a row, each
    checked against the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    layer = synth.make_layer(sp, [125, sp.M, B])
    x = synth.make_x(sp, B, [126, sp.M, B])
    d = fluxbin.DeviceLayer.from_host(layer)
    xd = torch.from_numpy(x).cuda()
    exact = oracle.linear(layer, x)
    for call in range(2):
        y = torch.full((B, sp.M), float("nan"), dtype=torch.float32, device="cuda")
        fluxbin.fluxbin_linear_static_scratch(d.desc, d.words, d.r, d.c, d.swords, d.rs, d.cs, d.idx, xd, B, y,
                                              fluxbin.FLAG_Y_FP32)
        torch.cuda.synchronize()
        got = y.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)), f"call {call}"
        close(got, exact, layer, x)

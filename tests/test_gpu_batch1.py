"""GPU parity of the batch-1, mu = 8 kernels against the fp64 oracle.

Large layers at batch 1 (M * N >= 2^27, or >= 2^25 with a workspace) run the
warp-specialised kernel (builder warps fill a two-stage table ring, lookup
warps consume it through mbarriers); FLUXBIN_FLAG_SEPARATE_TABLES runs the
table precompute as a kernel of its own followed by the lookup-only kernel
fed by bulk copies.  Both are compared with the oracle on every output row,
with and without a caller workspace (the plans differ: clusters or a split
through the workspace; mid-sized layers without one stay on the original
kernel), on ragged shapes and every base count the kernels are built for.
Same tolerance as the other parity tests; exact-arithmetic layers must match
bit for bit.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from lut_binary_basis_b200 import fluxbin, synth  # noqa: E402
from test_gpu_parity import assert_close, spec  # noqa: E402

pytestmark = pytest.mark.gpu

SEP = fluxbin.FLAG_SEPARATE_TABLES


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    fluxbin.fluxbin_device_status()
    yield
    assert fluxbin.fluxbin_device_status() == 0, "a bounded wait gave up"


def run(d, layer, x, flags, ws):
    y = torch.full((1, layer.spec.M), float("nan"), dtype=torch.float32, device="cuda")
    d.linear(torch.from_numpy(x).cuda(), y, fluxbin.FLAG_Y_FP32 | fluxbin.FLAG_EARLY_WEIGHTS | flags, ws)
    torch.cuda.synchronize()
    if ws is not None:
        n = fluxbin.fluxbin_workspace_bytes(layer.spec.M, 1) // 4
        assert int(ws[:n].abs().sum().item()) == 0, "workspace must be left zero-filled"
    return y.cpu().numpy().astype(np.float64)


LARGE = [
    spec(16411, 8200, 2, 2, 250, 8),      # ragged rows and columns
    spec(9000, 16000, 4, 1, 300, 8),
    spec(20000, 6711, 1, 0, 0, 8),
    spec(8195, 16384, 1, 4, 515, 8, outlier_frac=0.005),
]


@pytest.mark.parametrize("sp", LARGE, ids=lambda s: f"{s.M}x{s.N}_kb{s.Kb}_ks{s.Ks}")
def test_large_layers_every_row(sp):
    assert sp.M * sp.N >= 1 << 27
    _every_row(sp)


MID = [
    spec(11008, 4096, 2, 1, 205, 8),      # the 7B MLP shapes
    spec(4096, 11008, 2, 1, 550, 8),
    spec(6001, 5900, 1, 2, 300, 8),       # ragged rows and columns
    spec(8192, 4097, 4, 0, 0, 8),
]


@pytest.mark.parametrize("sp", MID, ids=lambda s: f"{s.M}x{s.N}_kb{s.Kb}_ks{s.Ks}")
def test_mid_layers_every_row(sp):
    assert (1 << 25) <= sp.M * sp.N < (1 << 27)
    _every_row(sp)


def _every_row(sp):
    layer = synth.make_layer(sp, [500, sp.M, sp.N])
    x = synth.make_x(sp, 1, [501, sp.M])
    ref = oracle.linear(layer, x)
    d = fluxbin.DeviceLayer.from_host(layer)
    for flags, ws in ((0, d.workspace(1)), (0, None), (SEP, d.workspace(1))):
        assert_close(run(d, layer, x, flags, ws), ref, layer, x)


@pytest.mark.parametrize("sp", [spec(2100, 777, 2, 1, 40, 8), spec(4096, 4096, 2, 1, 205, 8),
                                spec(33, 5000, 1, 2, 70, 8), spec(11008, 4096, 4, 4, 205, 8),
                                spec(3000, 1024, 2, 1, 1024, 8)],
                         ids=lambda s: f"{s.M}x{s.N}_kb{s.Kb}_ks{s.Ks}")
def test_separate_tables_small_layers(sp):
    """The precompute as its own kernel on layers of every size (odd unit
    counts, a split that starts inside a unit pair, every column salient)."""
    layer = synth.make_layer(sp, [510, sp.M, sp.N])
    x = synth.make_x(sp, 1, [511, sp.M])
    d = fluxbin.DeviceLayer.from_host(layer)
    assert_close(run(d, layer, x, SEP, d.workspace(1)), oracle.linear(layer, x), layer, x)


def test_exact_arithmetic_bit_exact_on_both_kernels():
    for i, sp in enumerate([spec(16400, 8192, 2, 1, 100, 8), spec(1030, 1500, 1, 2, 100, 8)]):
        layer = synth.make_exact_layer(sp, [520, i])
        x = synth.make_exact_x(sp, 1, [521, i])
        ref = oracle.linear(layer, x)
        d = fluxbin.DeviceLayer.from_host(layer)
        for flags in (0, SEP):
            got = run(d, layer, x, flags, d.workspace(1))
            assert np.array_equal(got, ref), f"case {i} flags {flags}: max diff {np.max(np.abs(got - ref))}"


def test_separate_tables_argument_errors():
    sp = spec(1000, 1024, 2, 1, 50, 8)
    layer = synth.make_layer(sp, [530])
    d = fluxbin.DeviceLayer.from_host(layer)
    x1 = torch.zeros((1, sp.N), dtype=torch.float16, device="cuda")
    y1 = torch.zeros((1, sp.M), dtype=torch.float32, device="cuda")
    small = fluxbin.new_workspace(sp.M, 1)
    for flags, ws, status in ((SEP, small, -6), (SEP, None, -6), (SEP | fluxbin.FLAG_PATH_TC, d.workspace(1), -1)):
        with pytest.raises(fluxbin.FluxbinError) as e:
            d.linear(x1, y1, fluxbin.FLAG_Y_FP32 | flags, ws)
        assert e.value.status == status
    x2 = torch.zeros((2, sp.N), dtype=torch.float16, device="cuda")
    y2 = torch.zeros((2, sp.M), dtype=torch.float32, device="cuda")
    with pytest.raises(fluxbin.FluxbinError) as e:
        d.linear(x2, y2, fluxbin.FLAG_Y_FP32 | SEP, d.workspace(2))
    assert e.value.status == -4
    blk = spec(256, 512, 2, 0, 0, 8, G=128)
    db = fluxbin.DeviceLayer.from_host(synth.make_layer(blk, [531]))
    with pytest.raises(fluxbin.FluxbinError) as e:
        db.linear(torch.zeros((1, 512), dtype=torch.float16, device="cuda"),
                  torch.zeros((1, 256), dtype=torch.float32, device="cuda"), fluxbin.FLAG_Y_FP32 | SEP,
                  fluxbin.new_workspace(256, 1, "cuda"))
    assert e.value.status == -4

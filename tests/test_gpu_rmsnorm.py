"""GPU parity of fluxbin_linear_rmsnorm: the table precompute fused with the
preceding RMS normalisation (LUT Tensor Core notes, Section 3.1.1), then the
lookups on the precomputed tables.

y is compared on every row with the fp64 oracle applied to the oracle's own
normalised row, x = h * gamma / sqrt(mean(h^2) + eps), with the tolerance of
the other parity tests (the max-abs bound taken with ||x||); the optional
normalised output x_out is the fp16 rounding of that x within one unit in
the last place.  Ragged shapes, gathered salient columns, every base count,
fp16 and fp32 y, accumulation; the argument errors of the entry point.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from lut_binary_basis_b200 import fluxbin, synth  # noqa: E402
from test_gpu_parity import assert_close, spec  # noqa: E402

pytestmark = pytest.mark.gpu

EPS = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    fluxbin.fluxbin_device_status()
    yield
    assert fluxbin.fluxbin_device_status() == 0, "a bounded wait gave up"


def inputs(sp, key):
    g = np.random.default_rng(key)
    h = (g.standard_normal(sp.N) * 2.5).astype(np.float16)
    h[g.choice(sp.N, max(1, sp.N // 200), replace=False)] *= np.float16(20)   # outlier channels
    gamma = g.uniform(0.5, 1.5, sp.N).astype(np.float16)
    return h, gamma


CASES = [
    spec(28672, 8192, 2, 2, 246, 8),       # the 70B MLP up shape
    spec(4096, 4096, 2, 1, 205, 8),
    spec(3001, 5003, 1, 2, 100, 8),        # ragged rows and columns
    spec(1000, 1024, 4, 0, 0, 8),
    spec(777, 2100, 2, 4, 300, 8),
]


@pytest.mark.parametrize("sp", CASES, ids=lambda s: f"{s.M}x{s.N}_kb{s.Kb}_ks{s.Ks}")
def test_fused_rmsnorm_every_row(sp):
    layer = synth.make_layer(sp, [700, sp.M, sp.N])
    h, gamma = inputs(sp, [701, sp.M])
    x = oracle.rmsnorm(h, gamma, EPS)
    ref = oracle.linear(layer, x[None, :])
    d = fluxbin.DeviceLayer.from_host(layer)
    hd, gd = torch.from_numpy(h).cuda(), torch.from_numpy(gamma).cuda()
    ws = d.workspace(1)
    y = torch.full((1, sp.M), float("nan"), dtype=torch.float32, device="cuda")
    x_out = torch.full((sp.N,), float("nan"), dtype=torch.float16, device="cuda")
    d.linear_rmsnorm(hd, gd, EPS, y, fluxbin.FLAG_Y_FP32 | fluxbin.FLAG_EARLY_WEIGHTS, ws, x_out)
    torch.cuda.synchronize()
    assert_close(y.cpu().numpy().astype(np.float64), ref, layer, x[None, :])
    xo = x_out.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(xo - x) <= np.abs(x) * 2.0 ** -10 + 2.0 ** -24), "x_out is not x rounded to fp16"
    n = fluxbin.fluxbin_workspace_bytes(sp.M, 1) // 4
    assert int(ws[:n].abs().sum().item()) == 0, "workspace must be left zero-filled"
    # fp16 y, accumulated onto a known start, no x_out
    y0 = torch.from_numpy(np.random.default_rng(702).standard_normal((1, sp.M)).astype(np.float16)).cuda()
    y16 = y0.clone()
    d.linear_rmsnorm(hd, gd, EPS, y16, fluxbin.FLAG_ACCUMULATE, ws)
    torch.cuda.synchronize()
    got = y16.cpu().numpy().astype(np.float64) - y0.cpu().numpy().astype(np.float64)
    # fp16 y: the output rounding adds half an ulp of |y| per row
    tol = np.abs(y16.cpu().numpy().astype(np.float64)) * 2.0 ** -11
    err = np.abs(got - ref) - tol
    assert np.linalg.norm(np.maximum(err, 0)) <= 2e-3 * np.linalg.norm(ref)


def test_fused_rmsnorm_matches_separate_tables_on_the_same_x():
    """The fused precompute and the plain one (FLUXBIN_FLAG_SEPARATE_TABLES)
    agree when the plain one is given the same x: gamma = 1, every entry of h
    +-4 and eps = 0 make x = +-1 (up to the rounding of 1/rms)."""
    sp = spec(2048, 2048, 2, 1, 128, 8)
    layer = synth.make_exact_layer(sp, [710])
    g = np.random.default_rng(711)
    h = np.where(g.random(sp.N) < 0.5, -4.0, 4.0).astype(np.float16)
    gamma = np.ones(sp.N, np.float16)
    d = fluxbin.DeviceLayer.from_host(layer)
    ws = d.workspace(1)
    y1 = torch.zeros((1, sp.M), dtype=torch.float32, device="cuda")
    y2 = torch.zeros((1, sp.M), dtype=torch.float32, device="cuda")
    d.linear_rmsnorm(torch.from_numpy(h).cuda(), torch.from_numpy(gamma).cuda(), 0.0, y1, fluxbin.FLAG_Y_FP32, ws)
    xs = (h / np.float16(4)).astype(np.float16)[None, :]
    d.linear(torch.from_numpy(xs).cuda(), y2, fluxbin.FLAG_Y_FP32 | fluxbin.FLAG_SEPARATE_TABLES, ws)
    torch.cuda.synchronize()
    a1, a2 = y1.cpu().numpy().astype(np.float64), y2.cpu().numpy().astype(np.float64)
    ref = oracle.linear(layer, xs)
    assert np.array_equal(a2, ref)
    assert np.max(np.abs(a1 - a2)) <= 1e-6 * np.max(np.abs(ref))


def test_fused_rmsnorm_argument_errors():
    sp = spec(1000, 1024, 2, 1, 50, 8)
    layer = synth.make_layer(sp, [720])
    d = fluxbin.DeviceLayer.from_host(layer)
    h = torch.zeros(sp.N, dtype=torch.float16, device="cuda")
    gm = torch.ones(sp.N, dtype=torch.float16, device="cuda")
    y = torch.zeros((1, sp.M), dtype=torch.float32, device="cuda")
    ws = d.workspace(1)
    small = fluxbin.new_workspace(sp.M, 1)

    def status(**kw):
        args = dict(h=h, gamma=gm, eps=EPS, y=y, flags=fluxbin.FLAG_Y_FP32, workspace=ws, x_out=None)
        args.update(kw)
        with pytest.raises(fluxbin.FluxbinError) as e:
            d.linear_rmsnorm(**args)
        return e.value.status

    assert status(workspace=small) == -6
    assert status(workspace=None) == -6
    assert status(eps=-1.0) == -1
    assert status(eps=float("nan")) == -1
    assert status(eps=float("inf")) == -1
    assert status(gamma=None) == -1
    assert status(x_out=h) == -1                                  # x_out overlaps h
    assert status(flags=fluxbin.FLAG_SEPARATE_TABLES) == -1
    assert status(flags=fluxbin.FLAG_PATH_TC) == -1
    for bad in (spec(256, 512, 2, 0, 0, 4), spec(256, 512, 2, 0, 0, 8, G=128)):
        db = fluxbin.DeviceLayer.from_host(synth.make_layer(bad, [721]))
        hb = torch.zeros(bad.N, dtype=torch.float16, device="cuda")
        gb = torch.ones(bad.N, dtype=torch.float16, device="cuda")
        yb = torch.zeros((1, bad.M), dtype=torch.float32, device="cuda")
        with pytest.raises(fluxbin.FluxbinError) as e:
            db.linear_rmsnorm(hb, gb, EPS, yb, fluxbin.FLAG_Y_FP32, db.workspace(1))
        assert e.value.status == -4

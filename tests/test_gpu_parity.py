"""GPU parity of the CUDA path (through the C-ABI) against the fp64 oracle.

Tolerance (floating point): per batch row b,
    relative L2 error  ||y - y_ref|| / ||y_ref||                <= 2e-3
    max abs error      max_i |y_i - y_ref_i| <= 1e-2 * ||x_b||_2 * max|r| * max|c|
(max over every base's row and column scales, both branches).  Cases with
small-integer activations and power-of-two scales are exact in fp32 and must
match bit for bit.
"""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from lut_binary_basis_b200 import fluxbin, synth  # noqa: E402
from lut_binary_basis_b200.synth import LayerSpec  # noqa: E402

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3
ABS_FACTOR = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


def run_linear(layer, x, flags=fluxbin.FLAG_Y_FP32, y0=None, dev="cuda"):
    d = fluxbin.DeviceLayer.from_host(layer, dev)
    B = x.shape[0]
    xd = torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    ydt = torch.float32 if flags & fluxbin.FLAG_Y_FP32 else torch.float16
    y = (torch.from_numpy(y0).to(dev).to(ydt) if y0 is not None
         else torch.full((B, layer.spec.M), float("nan"), dtype=ydt, device=dev))
    ws = fluxbin.new_workspace(layer.spec.M, B, dev)
    d.linear(xd, y, flags, ws)
    torch.cuda.synchronize()
    assert int(ws.abs().sum().item()) == 0, "workspace must be left zero-filled"
    return y.float().cpu().numpy().astype(np.float64)


def scale_bound(layer):
    mr = max(np.abs(layer.r.astype(np.float64)).max(initial=0), np.abs(layer.rs.astype(np.float64)).max(initial=0))
    mc = max(np.abs(layer.c.astype(np.float64)).max(initial=0), np.abs(layer.cs.astype(np.float64)).max(initial=0))
    return mr * mc


def assert_close(got, ref, layer, x):
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got))
    xn = np.linalg.norm(x.astype(np.float64), axis=1)
    bound = scale_bound(layer)
    for b in range(ref.shape[0]):
        nr = np.linalg.norm(ref[b])
        err = np.linalg.norm(got[b] - ref[b])
        assert err <= REL_L2 * nr + 1e-30, f"batch row {b}: relative L2 {err / max(nr, 1e-300):.3e}"
        mx = np.max(np.abs(got[b] - ref[b])) if ref.shape[1] else 0.0
        assert mx <= ABS_FACTOR * xn[b] * bound + 1e-30, f"batch row {b}: max abs {mx:.3e}"


def spec(M, N, Kb, Ks, n_sal, mu, G=0, **kw):
    return LayerSpec(f"t{M}x{N}", M, N, Kb, Ks, n_sal, mu, row_scale_group=G, **kw)


CASES = [
    (synth.layer_small(), 1),
    (spec(1000, 1000, 2, 1, 50, 8, outlier_frac=0.005), 1),
    (spec(1000, 1000, 2, 1, 50, 8, outlier_frac=0.005), 3),
    (spec(2100, 777, 2, 1, 40, 8), 1),
    (spec(2100, 777, 2, 2, 40, 8), 2),
    (spec(2100, 777, 1, 1, 300, 8), 5),
    (spec(2100, 777, 4, 2, 77, 8), 1),
    (spec(2100, 777, 4, 4, 77, 8), 2),
    (spec(1500, 1030, 2, 1, 60, 4), 1),
    (spec(1500, 1030, 2, 2, 60, 4), 4),
    (spec(1500, 1030, 1, 4, 60, 4), 7),
    (spec(1500, 1030, 4, 1, 60, 4), 16),
    (spec(700, 600, 2, 1, 30, 8), 16),
    (spec(33, 5, 1, 1, 2, 8), 2),
    (spec(1, 1, 1, 0, 0, 4), 1),
    (spec(3000, 256, 2, 1, 256, 8), 2),      # every column salient
    (spec(64, 2048, 2, 0, 0, 8, G=128), 1),  # block-wise row scales
    (spec(1100, 1024, 2, 1, 64, 4, G=128), 3),
    (spec(1100, 1024, 1, 0, 0, 8, G=256), 2),
    (spec(2100, 1024, 2, 2, 128, 8, G=128, sal_scale_group=16, sal_per_group=16), 1),  # 2.75-bit layout
    (spec(1100, 777, 2, 2, 120, 8, sal_scale_group=16), 3),
    (spec(1100, 777, 1, 1, 120, 8, sal_scale_group=8), 2),
    (spec(1100, 777, 2, 4, 120, 8, sal_scale_group=32), 1),
    (spec(900, 600, 2, 2, 100, 4, sal_scale_group=8), 2),
    (spec(900, 600, 1, 1, 100, 4, sal_scale_group=4), 1),
    (spec(900, 600, 4, 2, 100, 4, sal_scale_group=16), 1),
    (spec(256, 65536, 2, 1, 300, 8), 1),     # split wider than a cluster: workspace path
    (spec(100, 30000, 1, 2, 500, 4), 3),
    (spec(4096, 4096, 2, 1, 205, 8), 2),
]


@pytest.mark.parametrize("sp,B", CASES, ids=lambda v: getattr(v, "name", None) or f"B{v}")
def test_parity_random(sp, B):
    layer = synth.make_layer(sp, [77, sp.M, sp.N, B])
    x = synth.make_x(sp, B, [78, sp.M, sp.N, B])
    ref = oracle.linear(layer, x)
    got = run_linear(layer, x)
    assert_close(got, ref, layer, x)


@pytest.mark.parametrize("mu", [4, 8])
def test_exact_arithmetic_is_bit_exact(mu):
    for i, (sp, B) in enumerate([(spec(2100, 777, 2, 1, 40, mu), 3), (spec(1030, 1500, 1, 2, 100, mu), 1),
                                 (spec(300, 512, 2, 0, 0, mu, G=128), 2),
                                 (spec(700, 1024, 2, 2, 128, mu, G=128, sal_scale_group=2 * mu,
                                       sal_per_group=16), 2)]):
        layer = synth.make_exact_layer(sp, [80, i, mu])
        x = synth.make_exact_x(sp, B, [81, i, mu])
        ref = oracle.linear(layer, x)
        got = run_linear(layer, x)
        assert np.array_equal(got, ref), f"case {i}: max diff {np.max(np.abs(got - ref))}"


def test_fp16_output_and_accumulate():
    sp = spec(1000, 1000, 2, 1, 50, 8)
    layer = synth.make_layer(sp, [90])
    x = synth.make_x(sp, 2, [91])
    ref = oracle.linear(layer, x)
    got16 = run_linear(layer, x, flags=0)
    assert_close(got16, ref, layer, x)
    y0 = np.random.default_rng(5).standard_normal((2, sp.M)).astype(np.float32)
    got = run_linear(layer, x, flags=fluxbin.FLAG_Y_FP32 | fluxbin.FLAG_ACCUMULATE, y0=y0)
    assert_close(got - y0.astype(np.float64), ref, layer, x)
    y016 = y0.astype(np.float16)
    got = run_linear(layer, x, flags=fluxbin.FLAG_ACCUMULATE, y0=y016)
    assert_close(got - y016.astype(np.float64), ref, layer, x)


def test_early_weights_flag_same_result():
    sp = spec(2100, 777, 2, 1, 40, 8)
    layer = synth.make_layer(sp, [92])
    x = synth.make_x(sp, 1, [93])
    a = run_linear(layer, x)
    b = run_linear(layer, x, flags=fluxbin.FLAG_Y_FP32 | fluxbin.FLAG_EARLY_WEIGHTS)
    assert np.array_equal(a, b) or np.allclose(a, b, rtol=1e-6, atol=1e-4)


def test_lut_gemv_single_branch_with_gather():
    """The dense-branch entry point on a gathered column set equals the
    salient branch alone."""
    sp = spec(1500, 900, 1, 2, 130, 8)
    layer = synth.make_layer(sp, [94])
    x = synth.make_x(sp, 2, [95])
    dev = "cuda"
    words, swords = fluxbin.fluxbin_pack(fluxbin.LayerDesc.of(sp), layer.signs, layer.sal_signs, layer.sal_idx)
    sw = torch.from_numpy(swords.view(np.int32)).to(dev)
    rs = torch.from_numpy(layer.rs).to(dev)
    cs = torch.from_numpy(layer.cs).to(dev)
    idx = torch.from_numpy(layer.sal_idx).to(dev)
    xd = torch.from_numpy(x).to(dev)
    y = torch.zeros((2, sp.M), dtype=torch.float32, device=dev)
    ws = fluxbin.new_workspace(sp.M, 2, dev)
    fluxbin.fluxbin_lut_gemv(sp.M, sp.N, sp.n_sal, 2, 8, 0, sw, rs, cs, idx, xd, 2, y, fluxbin.FLAG_Y_FP32, ws)
    torch.cuda.synchronize()
    only_sal = dataclasses.replace(layer, c=np.zeros_like(layer.c))
    ref = oracle.linear(only_sal, x)
    assert_close(y.cpu().numpy().astype(np.float64), ref, only_sal, x)
    # an out-of-range column index contributes nothing
    bad = layer.sal_idx.copy()
    bad[5] = sp.N + 10
    fluxbin.fluxbin_lut_gemv(sp.M, sp.N, sp.n_sal, 2, 8, 0, sw, rs, cs, torch.from_numpy(bad).to(dev), xd, 2, y,
                             fluxbin.FLAG_Y_FP32, ws)
    torch.cuda.synchronize()
    cs0 = layer.cs.copy()
    cs0[:, 5] = 0
    ref0 = oracle.linear(dataclasses.replace(only_sal, cs=cs0), x)
    assert_close(y.cpu().numpy().astype(np.float64), ref0, only_sal, x)


def test_noop_and_errors_on_device():
    sp = spec(64, 128, 2, 1, 8, 8)
    layer = synth.make_layer(sp, [96])
    d = fluxbin.DeviceLayer.from_host(layer)
    x = torch.zeros((0, sp.N), dtype=torch.float16, device="cuda")
    y = torch.zeros((0, sp.M), dtype=torch.float32, device="cuda")
    d.linear(x, y, fluxbin.FLAG_Y_FP32, None)   # B = 0: nothing to do
    # a layer that would split its long rows through a workspace runs on
    # thread-block clusters (or unsplit) when the caller gives none
    big = spec(256, 65536, 2, 1, 205, 8)
    hl = synth.make_layer(big, [97])
    lb = fluxbin.DeviceLayer.from_host(hl)
    for B in (1, 2):
        xh = synth.make_x(big, B, [98, B])
        yb = torch.full((B, big.M), float("nan"), dtype=torch.float32, device="cuda")
        lb.linear(torch.from_numpy(xh).cuda(), yb, fluxbin.FLAG_Y_FP32, None)
        torch.cuda.synchronize()
        assert_close(yb.cpu().numpy().astype(np.float64), oracle.linear(hl, xh), hl, xh)
    # the tensor-core path always needs one
    xb = torch.zeros((16, big.N), dtype=torch.float16, device="cuda")
    yb = torch.zeros((16, big.M), dtype=torch.float32, device="cuda")
    with pytest.raises(fluxbin.FluxbinError) as e:
        lb.linear(xb, yb, fluxbin.FLAG_Y_FP32 | fluxbin.FLAG_PATH_TC, None)
    assert e.value.status == -6


# ---------------------------------------------------------------------------
# Full-size workloads, every output row compared with the oracle (the fp64
# oracle runs over rows in parallel on the host cores), in the launch
# configuration the benchmark times (packed words requested early, a caller
# workspace).  Each (layer, batch) runs on the path the library chooses; the
# batch-16 cases of the 70B-shaped layers also run forced onto the other path
# (tensor cores for mu = 8, the LUT path for mu = 4).
# ---------------------------------------------------------------------------

A, L, T = 0, fluxbin.FLAG_PATH_LUT, fluxbin.FLAG_PATH_TC

FULL = [
    # layer, workload id, [(batch, path flags)]
    (synth.layer_7b_proj(), 1, [(1, A)]),
    (synth.layers_7b_mlp()[0], 2, [(1, A), (2, A), (4, A), (8, A)]),
    (synth.layers_7b_mlp()[1], 2, [(1, A), (2, A), (4, A), (8, A)]),  # B = 1: split through the workspace
    (synth.layers_70b_mlp(8)[0], 3, [(1, A), (2, A), (16, A), (16, T)]),   # B >= 2: fp16-pair tables
    (synth.layers_70b_mlp(8)[1], 3, [(1, A), (16, A)]),
    (synth.layers_70b_mlp(4)[0], 3, [(1, A), (16, A), (16, L)]),
    (synth.layers_70b_mlp(4)[1], 3, [(1, A), (16, A)]),
    (synth.layers_7b_stack_linears()[0], 4, [(1, A)]),   # q: 2.75-bit, block-wise and grouped salient scales
    (synth.layers_7b_stack_linears()[4], 4, [(1, A)]),   # gate
    (synth.layers_7b_stack_linears()[6], 4, [(1, A)]),   # down
]


@pytest.mark.parametrize("sp,wid,runs", FULL, ids=lambda v: getattr(v, "name", None) or str(v))
def test_parity_full_size_every_row(sp, wid, runs):
    layer = synth.make_layer(sp, synth.layer_key(wid, 0, 0))
    d = fluxbin.DeviceLayer.from_host(layer)
    for B, path in runs:
        x = synth.make_x(sp, B, synth.x_key(wid, 0, 0, B))
        xd = torch.from_numpy(x).cuda()
        y = torch.full((B, sp.M), float("nan"), dtype=torch.float32, device="cuda")
        ws = fluxbin.new_workspace(sp.M, B)
        d.linear(xd, y, fluxbin.FLAG_Y_FP32 | fluxbin.FLAG_EARLY_WEIGHTS | path, ws)
        torch.cuda.synchronize()
        got = y.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)), f"B={B} path={path}"
        assert int(ws.abs().sum().item()) == 0, "workspace must be left zero-filled"
        assert_close(got, oracle.linear(layer, x), layer, x)


def test_long_rows_with_and_without_workspace():
    """A layer with long rows on few row groups (4096x11008 at batch 1) is
    split wider than a cluster through the caller's workspace; without one it
    runs on clusters.  Both match the oracle on every row, and the workspace
    is left zero."""
    sp = synth.layers_7b_mlp()[1]
    layer = synth.make_layer(sp, synth.layer_key(2, 0, 0))
    d = fluxbin.DeviceLayer.from_host(layer)
    x = synth.make_x(sp, 1, synth.x_key(2, 0, 0, 1))
    ref = oracle.linear(layer, x)
    xd = torch.from_numpy(x).cuda()
    outs = []
    for ws in (fluxbin.new_workspace(sp.M, 1), None):
        y = torch.full((1, sp.M), float("nan"), dtype=torch.float32, device="cuda")
        d.linear(xd, y, fluxbin.FLAG_Y_FP32, ws)
        torch.cuda.synchronize()
        got = y.cpu().numpy().astype(np.float64)
        assert_close(got, ref, layer, x)
        if ws is not None:
            assert int(ws.abs().sum().item()) == 0
        outs.append(got)
    # different split-K sums of the same products: equal within fp32 rounding
    assert np.allclose(outs[0], outs[1], rtol=1e-4, atol=1e-3 * np.abs(outs[1]).max())

"""GPU parity of the batch kernel on fp16-pair tables (batches of 2-16,
mu = 8, per-row scales) against the fp64 oracle.

Two batch rows share every table lookup: each table entry is stored once per
row pair as two fp16 values (table quantisation, LUT Tensor Core notes,
Section 3.1.3), consecutive steps are added in fp16 and accumulated in fp32.
The tolerance is the one of every other parity test (relative L2 2e-3,
max-abs 1e-2 * ||x||_2 * max|r| * max|c|); exact-arithmetic layers (small
integer activations, power-of-two scales: every table entry and pair sum is
an fp16 value) must match bit for bit.  Odd batches leave the last pair with
one row.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from lut_binary_basis_b200 import fluxbin, synth  # noqa: E402
from test_gpu_parity import assert_close, run_linear, spec  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    fluxbin.fluxbin_device_status()
    yield
    assert fluxbin.fluxbin_device_status() == 0, "a bounded wait gave up"


CASES = [
    (spec(4100, 4500, 2, 1, 225, 8), 2),
    (spec(2100, 777, 2, 1, 40, 8), 3),
    (spec(2100, 777, 1, 2, 300, 8), 5),
    (spec(1500, 3000, 4, 4, 150, 8, outlier_frac=0.005), 8),
    (spec(9000, 2048, 2, 0, 0, 8), 13),
    (spec(3000, 6000, 1, 1, 600, 8), 16),
    (spec(33, 9000, 2, 2, 700, 8), 4),      # one ragged row group, long rows
    (spec(17000, 1000, 4, 1, 90, 8), 7),    # many row groups
]


@pytest.mark.parametrize("sp,B", CASES, ids=lambda v: getattr(v, "name", None) or f"B{v}")
def test_pair_tables_random(sp, B):
    layer = synth.make_layer(sp, [600, sp.M, sp.N, B])
    x = synth.make_x(sp, B, [601, sp.M, B])
    ref = oracle.linear(layer, x)
    assert_close(run_linear(layer, x), ref, layer, x)
    # without a workspace the plan reduces in clusters (or not at all)
    d = fluxbin.DeviceLayer.from_host(layer)
    y = torch.full((B, sp.M), float("nan"), dtype=torch.float32, device="cuda")
    d.linear(torch.from_numpy(x).cuda(), y, fluxbin.FLAG_Y_FP32, None)
    torch.cuda.synchronize()
    assert_close(y.cpu().numpy().astype(np.float64), ref, layer, x)


@pytest.mark.parametrize("B", [2, 7, 16])
def test_pair_tables_exact_arithmetic_bit_exact(B):
    for i, sp in enumerate([spec(2100, 777, 2, 1, 40, 8), spec(5000, 4096, 1, 2, 300, 8)]):
        layer = synth.make_exact_layer(sp, [610, i, B])
        x = synth.make_exact_x(sp, B, [611, i, B], lo=-4, hi=4)
        ref = oracle.linear(layer, x)
        got = run_linear(layer, x)
        assert np.array_equal(got, ref), f"case {i}: max diff {np.max(np.abs(got - ref))}"


def test_pair_tables_fp16_output_accumulate_and_early_weights():
    sp = spec(5000, 4200, 2, 1, 210, 8)
    layer = synth.make_layer(sp, [620])
    x = synth.make_x(sp, 6, [621])
    ref = oracle.linear(layer, x)
    assert_close(run_linear(layer, x, flags=0), ref, layer, x)
    y0 = np.random.default_rng(7).standard_normal((6, sp.M)).astype(np.float32)
    got = run_linear(layer, x, flags=fluxbin.FLAG_Y_FP32 | fluxbin.FLAG_ACCUMULATE | fluxbin.FLAG_EARLY_WEIGHTS,
                     y0=y0)
    assert_close(got - y0.astype(np.float64), ref, layer, x)


def test_pair_tables_error_is_table_rounding_sized():
    """The fp16 tables cost accuracy of the order of fp16 rounding, not more:
    the error against the exact oracle stays within a few times the error of
    the oracle's own fp16-table evaluation."""
    sp = spec(4096, 4096, 2, 1, 205, 8, outlier_frac=0.005)
    layer = synth.make_layer(sp, [630])
    x = synth.make_x(sp, 4, [631])
    exact = oracle.linear(layer, x)
    q16 = oracle.lut_linear(layer, x, mu=8, tables="fp16")
    got = run_linear(layer, x)
    for b in range(4):
        e_gpu = np.linalg.norm(got[b] - exact[b])
        e_q = np.linalg.norm(q16[b] - exact[b])
        assert e_gpu <= 4 * e_q + 1e-6 * np.linalg.norm(exact[b])


@pytest.mark.parametrize("M,N,n_sal,B", [(16400, 9000, 8300, 1), (3000, 5000, 2600, 4), (2000, 3000, 1200, 7)],
                         ids=["batch1_large", "pairs_b4", "pairs_b7"])
def test_lut_gemv_gathered_branch_on_new_kernels(M, N, n_sal, B):
    """fluxbin_lut_gemv on a gathered column set (the salient branch alone,
    Virtual Columnar Mapping) through the warp-specialised batch-1 kernel
    (M * ncols >= 2^27) and the batch-pair kernel, with an out-of-range
    column index contributing nothing."""
    import dataclasses
    sp = spec(M, N, 1, 2, n_sal, 8)
    layer = synth.make_layer(sp, [640, M, B])
    x = synth.make_x(sp, B, [641, M, B])
    words, swords = fluxbin.fluxbin_pack(fluxbin.LayerDesc.of(sp), layer.signs, layer.sal_signs, layer.sal_idx)
    sw = torch.from_numpy(swords.view(np.int32)).cuda()
    rs, cs = torch.from_numpy(layer.rs).cuda(), torch.from_numpy(layer.cs).cuda()
    xd = torch.from_numpy(x).cuda()
    ws = fluxbin.new_workspace(M, B)
    only_sal = dataclasses.replace(layer, c=np.zeros_like(layer.c))
    for bad in (False, True):
        idx = layer.sal_idx.copy()
        cs_ref = layer.cs.copy()
        if bad:
            idx[7] = N + 3
            cs_ref[:, 7] = 0
        y = torch.full((B, M), float("nan"), dtype=torch.float32, device="cuda")
        fluxbin.fluxbin_lut_gemv(M, N, n_sal, 2, 8, 0, sw, rs, cs, torch.from_numpy(idx).cuda(), xd, B, y,
                                 fluxbin.FLAG_Y_FP32, ws)
        torch.cuda.synchronize()
        ref = oracle.linear(dataclasses.replace(only_sal, cs=cs_ref), x)
        assert_close(y.cpu().numpy().astype(np.float64), ref, only_sal, x)

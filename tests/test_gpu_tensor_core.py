"""GPU parity of the tensor-core path (fluxbin_tc.cuh) against the fp64 oracle.

The path is forced with FLUXBIN_FLAG_PATH_TC so that every batch size and
shape below runs on it; the default choice sends batches of 16 on layers above
4096x4096, and batches of 8 on layers of at least 16384 rows, there on its own
(the full-size 70B-shaped B = 16 cases of test_gpu_parity.py).  Same tolerance as the
LUT path; cases with small-integer activations and power-of-two scales are
exact (products exact in fp16, sums exact in fp32) and must match bit for bit.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from lut_binary_basis_b200 import fluxbin, synth  # noqa: E402
from test_gpu_parity import assert_close, run_linear, spec  # noqa: E402

pytestmark = pytest.mark.gpu

TC = fluxbin.FLAG_Y_FP32 | fluxbin.FLAG_PATH_TC


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    fluxbin.fluxbin_device_status()   # start clean
    yield
    assert fluxbin.fluxbin_device_status() == 0, "a tensor-core wait gave up"


CASES = [
    (spec(256, 512, 2, 1, 40, 8), 16),
    (spec(1000, 777, 1, 2, 100, 8), 8),      # ragged rows and columns, two salient bases
    (spec(300, 2048, 4, 4, 64, 8), 5),
    (spec(130, 300, 2, 0, 0, 8), 1),         # no salient branch, one batch row
    (spec(33, 8192, 2, 2, 246, 8), 12),      # one ragged tile, units split over many items
    (spec(4096, 4096, 2, 1, 205, 8), 16),
    (spec(11008, 4096, 2, 1, 205, 8), 3),
    (spec(300, 1024, 2, 2, 64, 4), 16),      # mu = 4
    (spec(1000, 777, 1, 1, 100, 4), 8),
    (spec(257, 2048, 4, 4, 33, 4), 16),
    (spec(28672 // 8, 8192, 2, 2, 246, 4), 16),
]


@pytest.mark.parametrize("sp,B", CASES, ids=lambda v: getattr(v, "name", None) or f"B{v}")
def test_tc_parity_random(sp, B):
    layer = synth.make_layer(sp, [177, sp.M, sp.N, B])
    x = synth.make_x(sp, B, [178, sp.M, sp.N, B])
    ref = oracle.linear(layer, x)
    got = run_linear(layer, x, flags=TC)
    assert_close(got, ref, layer, x)


def test_tc_exact_arithmetic_is_bit_exact():
    for i, (sp, B) in enumerate([(spec(2100, 777, 2, 1, 40, 8), 16), (spec(1030, 1500, 1, 2, 100, 8), 9),
                                 (spec(200, 4096, 4, 1, 33, 8), 4), (spec(700, 1500, 2, 2, 90, 4), 16),
                                 (spec(130, 600, 4, 4, 20, 4), 3)]):
        layer = synth.make_exact_layer(sp, [180, i])
        x = synth.make_exact_x(sp, B, [181, i])
        ref = oracle.linear(layer, x)
        got = run_linear(layer, x, flags=TC)
        assert np.array_equal(got, ref), f"case {i}: max diff {np.max(np.abs(got - ref))}"


def test_tc_fp16_output_and_accumulate():
    sp = spec(1000, 1000, 2, 1, 50, 8)
    layer = synth.make_layer(sp, [190])
    x = synth.make_x(sp, 16, [191])
    ref = oracle.linear(layer, x)
    assert_close(run_linear(layer, x, flags=fluxbin.FLAG_PATH_TC), ref, layer, x)
    y0 = np.random.default_rng(6).standard_normal((16, sp.M)).astype(np.float32)
    got = run_linear(layer, x, flags=TC | fluxbin.FLAG_ACCUMULATE, y0=y0)
    assert_close(got - y0.astype(np.float64), ref, layer, x)


def test_tc_and_lut_agree_and_default_choice():
    sp = spec(2048, 3000, 2, 2, 150, 8)
    layer = synth.make_layer(sp, [192])
    x = synth.make_x(sp, 16, [193])
    ref = oracle.linear(layer, x)
    for flags in (TC, fluxbin.FLAG_Y_FP32 | fluxbin.FLAG_PATH_LUT, fluxbin.FLAG_Y_FP32,
                  TC | fluxbin.FLAG_EARLY_WEIGHTS):
        assert_close(run_linear(layer, x, flags=flags), ref, layer, x)


def test_tc_refuses_what_it_does_not_cover():
    x = torch.zeros((16, 512), dtype=torch.float16, device="cuda")
    y = torch.zeros((16, 256), dtype=torch.float32, device="cuda")
    for sp, status in ((spec(256, 512, 2, 0, 0, 8, G=128), -4),     # block-wise row scales
                       (spec(256, 512, 2, 2, 256, 8, sal_scale_group=128), -4),  # block-wise salient scales
                       (spec(256, 512, 2, 2, 64, 8, sal_scale_group=16), -4)):   # grouped salient scales
        d = fluxbin.DeviceLayer.from_host(synth.make_layer(sp, [194]))
        with pytest.raises(fluxbin.FluxbinError) as e:
            d.linear(x, y, TC, fluxbin.new_workspace(sp.M, 16))
        assert e.value.status == status
    sp = spec(256, 512, 2, 1, 40, 8)
    d = fluxbin.DeviceLayer.from_host(synth.make_layer(sp, [195]))
    with pytest.raises(fluxbin.FluxbinError) as e:
        d.linear(x, y, TC, None)
    assert e.value.status == -6
    with pytest.raises(fluxbin.FluxbinError) as e:
        d.linear(x, y, TC | fluxbin.FLAG_PATH_LUT, fluxbin.new_workspace(sp.M, 16))
    assert e.value.status == -1


def test_tc_single_branch_with_gather():
    """fluxbin_lut_gemv on a gathered column set (the salient branch alone) on the tensor cores."""
    import dataclasses
    sp = spec(1500, 900, 1, 2, 130, 8)
    layer = synth.make_layer(sp, [196])
    x = synth.make_x(sp, 16, [197])
    words, swords = fluxbin.fluxbin_pack(fluxbin.LayerDesc.of(sp), layer.signs, layer.sal_signs, layer.sal_idx)
    dev = "cuda"
    sw = torch.from_numpy(swords.view(np.int32)).to(dev)
    rs, cs = torch.from_numpy(layer.rs).to(dev), torch.from_numpy(layer.cs).to(dev)
    idx = torch.from_numpy(layer.sal_idx).to(dev)
    y = torch.zeros((16, sp.M), dtype=torch.float32, device=dev)
    fluxbin.fluxbin_lut_gemv(sp.M, sp.N, sp.n_sal, 2, 8, 0, sw, rs, cs, idx, torch.from_numpy(x).to(dev), 16, y,
                             TC, fluxbin.new_workspace(sp.M, 16, dev))
    torch.cuda.synchronize()
    only_sal = dataclasses.replace(layer, c=np.zeros_like(layer.c))
    assert_close(y.cpu().numpy().astype(np.float64), oracle.linear(only_sal, x), only_sal, x)

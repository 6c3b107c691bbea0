"""The tensor-core kernel's bounded waits, made to run out on purpose.

FLUXBIN_FLAG_TEST_WAIT_TIMEOUT (a test hook) keeps the preparing warps from
ever reporting a buffer ready and shortens every mbarrier wait to a few
polls.  The issuing thread's first wait therefore gives up before any matrix
operation is issued; the call must then report the failure through
fluxbin_device_status (bit 0), write NaN outputs, release its tensor memory
(bit 1 stays clear) and leave the workspace zero-filled, and the context
must stay usable: the next ordinary call on the same layer is correct.
Nothing faults or hangs: every wait ends by its poll limit.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from lut_binary_basis_b200 import fluxbin, synth  # noqa: E402
from test_gpu_parity import assert_close, spec  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("sp,B", [(spec(1000, 1024, 2, 1, 50, 8), 16), (spec(4096, 4096, 2, 2, 123, 4), 4)],
                         ids=["mu8_b16", "mu4_b4_split"])
def test_tc_wait_timeout_reports_and_recovers(sp, B):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    assert fluxbin.fluxbin_device_status() == 0
    layer = synth.make_layer(sp, [400, sp.M])
    x = synth.make_x(sp, B, [401, sp.M])
    d = fluxbin.DeviceLayer.from_host(layer)
    xd = torch.from_numpy(x).cuda()
    ws = fluxbin.new_workspace(sp.M, B)
    y = torch.zeros((B, sp.M), dtype=torch.float32, device="cuda")
    hook = fluxbin.FLAG_Y_FP32 | fluxbin.FLAG_PATH_TC | fluxbin.FLAG_TEST_WAIT_TIMEOUT
    d.linear(xd, y, hook, ws)
    torch.cuda.synchronize()
    assert fluxbin.fluxbin_device_status() == 1, "the give-up path must report bit 0 only"
    assert fluxbin.fluxbin_device_status() == 0, "reading the status clears it"
    assert torch.isnan(y).all().item()
    assert int(ws.abs().sum().item()) == 0
    # the hook is refused without the tensor-core path
    with pytest.raises(fluxbin.FluxbinError) as e:
        d.linear(xd, y, fluxbin.FLAG_Y_FP32 | fluxbin.FLAG_TEST_WAIT_TIMEOUT, ws)
    assert e.value.status == -1
    # the context is intact: the same layer runs correctly afterwards
    y.zero_()
    d.linear(xd, y, fluxbin.FLAG_Y_FP32 | fluxbin.FLAG_PATH_TC, ws)
    torch.cuda.synchronize()
    assert fluxbin.fluxbin_device_status() == 0
    assert_close(y.cpu().numpy().astype(np.float64), oracle.linear(layer, x), layer, x)

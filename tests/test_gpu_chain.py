"""A decode-style chain of dependent layers captured in one CUDA graph,
checked against the oracle evaluating the same chain.

Every call runs with FLUXBIN_FLAG_EARLY_WEIGHTS (programmatic dependent
launch: each kernel starts and requests its packed signs while its
predecessor on the stream is still running) and all calls share one
workspace, as the decoder-stack benchmark runs them.  The chain mixes the
kernels and launch plans the library uses: the original kernel with a split
through the workspace (4096x4096, and the 2.75-bit stack layout with
block-wise row scales and grouped salient scales), the warp-specialised
batch-1 kernel (11008x4096, 4096x11008, 32768x4096), the table precompute
fused with an RMS normalisation of the previous layer's output followed by
the lookup-only kernel, a mu = 4 layer, and at batch 16 two tensor-core
layers (forced) followed by the batch-pair kernel.  Each layer reads the
previous layer's fp16 output as its activations, so a kernel that read its
input before its predecessor finished writing it would be caught.  The graph
is replayed twice and every output of every replay is compared with the
oracle chain (fp64 layers, outputs rounded to fp16 between layers as the
kernels do; the oracle's RMS normalisation for the fused layer, which has a
workspace of its own because it leaves its table buffer filled).  Column scales are divided by a power of two near sqrt(N) (an
exact rescaling of the fp16 values) so activations keep their magnitude
along the chain instead of overflowing fp16.

Context: the pages run the decode kernels under CUDA graphs (news article),
and the whole layer is the GEMV (FluxBin summary, Section 3).
"""
import dataclasses
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from lut_binary_basis_b200 import fluxbin, synth  # noqa: E402
from lut_binary_basis_b200.synth import LayerSpec  # noqa: E402
from test_gpu_parity import assert_close  # noqa: E402

pytestmark = pytest.mark.gpu


def _shrink(layer):
    """Column scales (both branches) divided by 2^ceil(log2(sqrt(N)))."""
    f = 2.0 ** -math.ceil(math.log2(math.sqrt(layer.spec.N)))
    return dataclasses.replace(layer, c=(layer.c.astype(np.float64) * f).astype(np.float16),
                               cs=(layer.cs.astype(np.float64) * f).astype(np.float16))


NORM, TC = "norm", "tc"
EPS = 1e-5


def _chains():
    """Per chain: (layer specs, batch, per-layer mode: None, NORM or TC)."""
    b1 = [
        (synth.layer_7b_proj(), None),                             # 4096x4096: workspace split
        (synth.layers_7b_mlp()[0], None),                          # 11008x4096: warp-specialised
        (synth.layers_7b_mlp()[1], None),                          # 4096x11008: warp-specialised
        (LayerSpec("t4096x4096n", 4096, 4096, 2, 1, synth.salient_count(4096, 0.05), 8), NORM),
        (synth.layers_7b_stack_linears()[0], None),                # 2.75-bit: G = 128, grouped salient scales
        (LayerSpec("t32768x4096", 32768, 4096, 2, 2, synth.salient_count(4096, 0.03), 8), None),
        (LayerSpec("t4096x32768_mu4", 4096, 32768, 2, 2, synth.salient_count(32768, 0.03), 4), None),
    ]
    b16 = [
        (LayerSpec("t8192x4096", 8192, 4096, 2, 1, synth.salient_count(4096, 0.05), 8), TC),
        (LayerSpec("t4096x8192", 4096, 8192, 2, 1, synth.salient_count(8192, 0.05), 8), TC),
        (LayerSpec("t4096x4096", 4096, 4096, 2, 2, synth.salient_count(4096, 0.03), 8), None),   # batch pairs
    ]
    return [([sp for sp, _ in b1], 1, [m for _, m in b1]), ([sp for sp, _ in b16], 16, [m for _, m in b16])]


def test_graph_of_dependent_layers_matches_oracle():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    dev = "cuda"
    chains = []
    max_m = 0
    for ci, (specs, B, modes) in enumerate(_chains()):
        layers = [_shrink(synth.make_layer(sp, [300 + ci, i])) for i, sp in enumerate(specs)]
        for a, b in zip(specs, specs[1:]):
            assert b.N == a.M
        gammas = [np.random.default_rng([320 + ci, i]).uniform(0.5, 1.5, sp.N).astype(np.float16)
                  if m == NORM else None for i, (sp, m) in enumerate(zip(specs, modes))]
        x0 = synth.make_x(specs[0], B, [310 + ci])
        # the oracle chain: fp64 layers, fp16 between layers; the fused layer
        # normalises its input row first
        xs_ref, ys_ref = [], []
        h = x0.astype(np.float64)
        for lay, m, gm in zip(layers, modes, gammas):
            x = oracle.rmsnorm(h[0], gm, EPS)[None, :] if m == NORM else h
            y = oracle.linear(lay, x)
            xs_ref.append(x)
            ys_ref.append(y)
            h = y.astype(np.float16).astype(np.float64)
        dls = [fluxbin.DeviceLayer.from_host(lay, dev) for lay in layers]
        gds = [torch.from_numpy(gm).to(dev) if gm is not None else None for gm in gammas]
        bufs = [torch.from_numpy(x0).to(dev)] + [torch.full((B, sp.M), float("nan"), dtype=torch.float16,
                                                             device=dev) for sp in specs]
        # the fused layer leaves its table buffer filled: it gets a workspace of its own
        gds = [(gd, d.workspace(1)) if gd is not None else None for gd, d in zip(gds, dls)]
        chains.append((layers, dls, bufs, xs_ref, ys_ref, modes, gds))
        max_m = max(max_m, max(sp.M for sp in specs))
    ws = fluxbin.new_workspace(max_m, 16, dev)
    flags = fluxbin.FLAG_EARLY_WEIGHTS    # fp16 outputs, as a decode chain keeps them

    stream = torch.cuda.Stream()

    def step():
        for layers, dls, bufs, _, _, modes, gds in chains:
            for i, d in enumerate(dls):
                if modes[i] == NORM:
                    d.linear_rmsnorm(bufs[i][0], gds[i][0], EPS, bufs[i + 1], flags, gds[i][1], None, stream)
                elif modes[i] == TC:
                    d.linear(bufs[i], bufs[i + 1], flags | fluxbin.FLAG_PATH_TC, ws, stream)
                else:
                    d.linear(bufs[i], bufs[i + 1], flags, ws, stream)

    with torch.cuda.stream(stream):
        step()                      # eager run: kernel attributes are set outside the capture
    stream.synchronize()
    for _, _, bufs, _, _, _, _ in chains:
        for b in bufs[1:]:
            b.fill_(float("nan"))
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    for replay in range(2):
        for _, _, bufs, _, _, _, _ in chains:
            for b in bufs[1:]:
                b.fill_(float("nan"))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        assert int(ws.abs().sum().item()) == 0, "workspace must be left zero-filled"
        assert fluxbin.fluxbin_device_status() == 0, "a bounded wait gave up"
        for layers, _, bufs, xs_ref, ys_ref, _, _ in chains:
            for i, lay in enumerate(layers):
                got = bufs[i + 1].float().cpu().numpy().astype(np.float64)
                assert np.all(np.isfinite(got)), f"replay {replay}, {lay.spec.name}: non-finite output"
                assert_close(got, ys_ref[i], lay, xs_ref[i])
    del g

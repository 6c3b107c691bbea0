"""Seeded synthetic inputs for FluxBin layers.

This module only draws random numbers and arranges them into plain arrays
(signs as int8 +-1, fp16 scales, fp16 activations, int32 salient column
lists).  It holds none of the method's arithmetic, so both the fp64 oracle
and the CUDA path consume its output without sharing any computation.

Shapes and distributions follow the FluxBin workloads:
  * sign bits are iid Bernoulli(0.5) (the +-1 bases of the decoupled
    row-column binary decomposition, "FluxBin" paper summary, Section 3
    "Quantization");
  * row and column scales are LogNormal(0, 0.3) rounded to fp16; every base
    after the first global one (and every salient base) is additionally
    multiplied by 0.3, since later bases and the salient refinement
    approximate a residual ("FluxBin" summary, Section 3 "Salient-Aware
    Hybrid Bases");
  * activations are fp16 N(0, 1), optionally with a seeded set of outlier
    channels multiplied by a constant in every batch row;
  * salient columns are a seeded uniform choice without replacement, sorted,
    or s columns chosen at random inside every group of G columns (the
    group-structured saliency of the summary's Section 3 "Structural
    Saliency Search" and Appendix B).

Randomness: numpy PCG64 seeded from SeedSequence([workload id, layer,
linear id, seed]); each tensor takes its own spawned child in the fixed
order listed in ``_STREAMS``.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np

_STREAMS = ("signs", "r", "c", "sal_idx", "sal_signs", "rs", "cs", "x", "outliers")


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    """Shape and structure of one FluxBin linear layer (W is M x N)."""

    name: str
    M: int
    N: int
    Kb: int            # global binary bases
    Ks: int            # salient refinement bases (0: no salient branch)
    n_sal: int         # salient columns (ignored when Ks == 0)
    mu: int            # LUT sub-vector length
    row_scale_group: int = 0   # 0: one row scale per row; G: one per G-column block
    sal_scale_group: int = 0   # 0: one salient row scale per row; s: one per s salient columns
    sal_per_group: int = 0     # >0: choose this many salient columns inside every row_scale_group block
    outlier_frac: float = 0.0  # fraction of activation channels that are outliers
    outlier_mult: float = 20.0

    @property
    def has_salient(self) -> bool:
        return self.Ks > 0 and self.n_sal > 0


@dataclasses.dataclass
class LayerData:
    """Host arrays for one layer, in the layouts the C-ABI documents."""

    spec: LayerSpec
    signs: np.ndarray            # int8 [Kb][M][N], values +-1
    r: np.ndarray                # fp16 [Kb][M] or [Kb][ceil(N/G)][M]
    c: np.ndarray                # fp16 [Kb][N]
    sal_idx: np.ndarray          # int32 [n_sal], strictly increasing
    sal_signs: np.ndarray        # int8 [Ks][M][n_sal]
    rs: np.ndarray               # fp16 [Ks][M] or [Ks][ceil(n_sal/s)][M]
    cs: np.ndarray               # fp16 [Ks][n_sal]


def round_half_up(v: float) -> int:
    return int(np.floor(v + 0.5))


def salient_count(N: int, frac: float) -> int:
    """Number of salient columns for a fraction of N (4096 * 5% -> 205)."""
    return round_half_up(N * frac)


def _rng(key: Sequence[int]) -> Dict[str, np.random.Generator]:
    ss = np.random.SeedSequence(list(key))
    children = ss.spawn(len(_STREAMS))
    return {name: np.random.Generator(np.random.PCG64(ch)) for name, ch in zip(_STREAMS, children)}


def _signs(g: np.random.Generator, shape) -> np.ndarray:
    """iid fair +-1 signs: the bits of the generator's raw 64-bit output, each
    byte spread to eight sign bytes by one multiply (bit t -> byte 7-t)."""
    n = int(np.prod(shape))
    raw = g.bit_generator.random_raw((n + 63) // 64).astype(np.uint64)
    byt = raw.view(np.uint8)[: (n + 7) // 8].astype(np.uint64)
    spread = ((byt * np.uint64(0x8040201008040201)) & np.uint64(0x8080808080808080)) >> np.uint64(7)
    s = spread.view(np.int8)[:n]
    s = s * np.int8(2)
    s -= np.int8(1)
    return s.reshape(shape)


def _lognormal_fp16(g: np.random.Generator, shape, sigma: float = 0.3) -> np.ndarray:
    return np.exp(sigma * g.standard_normal(shape)).astype(np.float16)


def _base_factor(n: int, first_full: bool) -> np.ndarray:
    f = np.full((n, 1), 0.3, dtype=np.float64)
    if first_full and n > 0:
        f[0] = 1.0
    return f


def make_layer(spec: LayerSpec, key: Sequence[int]) -> LayerData:
    """Draw one layer's signs, scales and salient structure from ``key``."""
    g = _rng(key)
    M, N, Kb = spec.M, spec.N, spec.Kb
    signs = _signs(g["signs"], (Kb, M, N))
    ngr = (N + spec.row_scale_group - 1) // spec.row_scale_group if spec.row_scale_group else 0
    r_shape = (Kb, ngr, M) if ngr else (Kb, M)
    r = _lognormal_fp16(g["r"], r_shape).astype(np.float64)
    r = (r.reshape(Kb, -1) * _base_factor(Kb, True)).reshape(r_shape).astype(np.float16)
    c = (_lognormal_fp16(g["c"], (Kb, N)).astype(np.float64) * _base_factor(Kb, True)).astype(np.float16)

    Ks = spec.Ks if spec.has_salient else 0
    if Ks:
        if spec.sal_per_group:
            G = spec.row_scale_group
            assert G > 0 and N % G == 0
            idx = []
            for blk in range(N // G):
                pick = g["sal_idx"].choice(G, size=spec.sal_per_group, replace=False)
                idx.append(blk * G + np.sort(pick))
            sal_idx = np.concatenate(idx).astype(np.int32)
        else:
            sal_idx = np.sort(g["sal_idx"].choice(N, size=spec.n_sal, replace=False)).astype(np.int32)
        n_sal = int(sal_idx.size)
        assert n_sal == spec.n_sal, (n_sal, spec.n_sal)
        sal_signs = _signs(g["sal_signs"], (Ks, M, n_sal))
        ngs = (n_sal + spec.sal_scale_group - 1) // spec.sal_scale_group if spec.sal_scale_group else 0
        rs_shape = (Ks, ngs, M) if ngs else (Ks, M)
        rs = (_lognormal_fp16(g["rs"], rs_shape).astype(np.float64) * 0.3).astype(np.float16)
        cs = (_lognormal_fp16(g["cs"], (Ks, n_sal)).astype(np.float64) * 0.3).astype(np.float16)
    else:
        sal_idx = np.zeros((0,), np.int32)
        sal_signs = np.zeros((0, M, 0), np.int8)
        rs = np.zeros((0, M), np.float16)
        cs = np.zeros((0, 0), np.float16)
    return LayerData(spec, signs, r, c, sal_idx, sal_signs, rs, cs)


def make_x(spec: LayerSpec, B: int, key: Sequence[int]) -> np.ndarray:
    """fp16 activations [B][N], N(0,1) with optional outlier channels."""
    g = _rng(key)
    x = g["x"].standard_normal((B, spec.N))
    n_out = round_half_up(spec.outlier_frac * spec.N) if spec.outlier_frac > 0 else 0
    if n_out:
        ch = g["outliers"].choice(spec.N, size=n_out, replace=False)
        x[:, ch] *= spec.outlier_mult
    return x.astype(np.float16)


# ----------------------------------------------------------------------------
# Exact-arithmetic inputs: small integers and powers of two, so that every
# partial sum is exactly representable in fp32 and results can be compared
# bit for bit.
# ----------------------------------------------------------------------------

def make_exact_layer(spec: LayerSpec, key: Sequence[int], unit_scales: bool = False) -> LayerData:
    d = make_layer(spec, key)
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key) + [99])))
    pow2 = np.array([0.5, 1.0, 2.0], dtype=np.float16)

    def pick(shape):
        if unit_scales:
            return np.ones(shape, np.float16)
        return pow2[g.integers(0, 3, size=shape)]

    return dataclasses.replace(
        d,
        r=pick(d.r.shape), c=pick(d.c.shape),
        rs=pick(d.rs.shape), cs=pick(d.cs.shape),
    )


def make_exact_x(spec: LayerSpec, B: int, key: Sequence[int], lo: int = -8, hi: int = 8) -> np.ndarray:
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key) + [7])))
    return g.integers(lo, hi + 1, size=(B, spec.N)).astype(np.float16)


# ----------------------------------------------------------------------------
# The workloads (shapes, base counts, salient fractions, sub-vector lengths).
# ----------------------------------------------------------------------------

def layer_small() -> LayerSpec:
    """256 x 256, one global base, mu = 4, no salient branch."""
    return LayerSpec("small_256x256", 256, 256, Kb=1, Ks=0, n_sal=0, mu=4)


def layer_7b_proj() -> LayerSpec:
    """LLaMA-2-7B-shaped 4096 x 4096 projection: 2 global bases, 5% salient
    columns (205) with 1 extra base, 0.5% outlier channels x20, mu = 8."""
    return LayerSpec("llama7b_proj_4096x4096", 4096, 4096, Kb=2, Ks=1,
                     n_sal=salient_count(4096, 0.05), mu=8, outlier_frac=0.005)


def layers_7b_mlp(mu: int = 8) -> List[LayerSpec]:
    """LLaMA-2-7B MLP: gate/up 11008 x 4096 and down 4096 x 11008."""
    return [
        LayerSpec("llama7b_gate_up_11008x4096", 11008, 4096, Kb=2, Ks=1,
                  n_sal=salient_count(4096, 0.05), mu=mu),
        LayerSpec("llama7b_down_4096x11008", 4096, 11008, Kb=2, Ks=1,
                  n_sal=salient_count(11008, 0.05), mu=mu),
    ]


def layers_70b_mlp(mu: int = 8) -> List[LayerSpec]:
    """70B-shaped MLP: up 28672 x 8192 and down 8192 x 28672, 3% salient
    columns with 2 extra bases, 0.5% outlier channels."""
    return [
        LayerSpec(f"llama70b_up_28672x8192_mu{mu}", 28672, 8192, Kb=2, Ks=2,
                  n_sal=salient_count(8192, 0.03), mu=mu, outlier_frac=0.005),
        LayerSpec(f"llama70b_down_8192x28672_mu{mu}", 8192, 28672, Kb=2, Ks=2,
                  n_sal=salient_count(28672, 0.03), mu=mu, outlier_frac=0.005),
    ]


def layers_7b_stack_linears() -> List[LayerSpec]:
    """The seven linears of one LLaMA-2-7B decoder layer in the mixed
    ~2.75-bit format: 2 global bases with block-wise (G = 128) row scales,
    s = 16 salient columns per 128-column block with 2 extra bases and one
    salient row scale per block."""
    out = []
    for name, M, N in (("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                       ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)):
        out.append(LayerSpec(f"llama7b_{name}_{M}x{N}_2b_s16_g128", M, N, Kb=2, Ks=2,
                             n_sal=(N // 128) * 16, mu=8, row_scale_group=128,
                             sal_scale_group=16, sal_per_group=16))
    return out


WORKLOADS = {
    0: ("small_256x256_b1", [layer_small()], [1]),
    1: ("llama7b_proj_4096x4096_b1", [layer_7b_proj()], [1]),
    2: ("llama7b_mlp_b1_2_4_8", layers_7b_mlp(), [1, 2, 4, 8]),
    3: ("llama70b_mlp_mu8_mu4_b1_16", layers_70b_mlp(8) + layers_70b_mlp(4), [1, 16]),
    4: ("llama7b_stack_32x7_275bit_b1", layers_7b_stack_linears(), [1]),
}


def layer_key(workload_id: int, layer: int, linear_id: int, seed: int = 0) -> List[int]:
    return [workload_id, layer, linear_id, seed]


def x_key(workload_id: int, layer: int, linear_id: int, B: int, seed: int = 0) -> List[int]:
    return [workload_id, layer, linear_id, seed, 1000 + B]


def scaled_spec(spec: LayerSpec, M: Optional[int] = None, N: Optional[int] = None,
                n_sal: Optional[int] = None, **kw) -> LayerSpec:
    """A smaller layer with the same structure (for oracle-sized parity runs)."""
    return dataclasses.replace(spec, M=M if M is not None else spec.M, N=N if N is not None else spec.N,
                               n_sal=n_sal if n_sal is not None else spec.n_sal, **kw)

"""Storage, shared-memory and throughput accounting from the FluxBin pages --
TEST INFRASTRUCTURE ONLY (pinned by the printed figures in tests/golden/).

  * Appendix C.2 "Storage Consumption Analysis": columns are grouped in
    blocks of G, s salient columns are chosen per block (N_sal = N/G * s);
    Kb global and Ks salient bases are stored as bits, and every scale and
    index as fp16.  The global base stores dense bits, column scales and
    block-wise row scales; the salient branch stores its bits, scales and
    the index of each salient column.
  * Appendix E.2 "Shared Memory Footprint Analysis": the kernel's shared
    memory holds the batch-specific, scale-fused tables plus an accumulation
    buffer of one partial sum per row of the tile, per base and per batch row.
  * Appendix E.3: effective TFLOPS is the equivalent fp16 work 2*M*N*B per
    second, counting the salient branch's columns too.
"""
from __future__ import annotations


def abw_leading(Kb: int, Ks: int, G: int, s: int) -> float:
    """Average bits per weight to leading order in 1/M and 1/N:
    Kb bits of global signs, Ks*s/G bits of salient signs, and 16 bits for
    each of the (Kb + Ks) fp16 row scales of a G-column block."""
    return Kb + Ks * s / G + 16.0 * (Kb + Ks) / G


def abw_exact(M: int, N: int, Kb: int, Ks: int, G: int, s: int) -> float:
    """Average bits per weight of one M x N layer, every stored item counted:
    global signs, salient signs, block-wise row scales for both branches,
    per-column scales for both branches and one fp16 index per salient column."""
    n_sal = (N // G) * s
    bits = Kb * M * N + Ks * M * n_sal
    bits += 16 * (Kb + Ks) * M * (N // G)
    bits += 16 * (Kb * N + Ks * n_sal)
    bits += 16 * n_sal
    return bits / (M * N)


def lut_smem_bytes(Kb: int, batch: int, Ktile: int, mu: int, Mtile: int, entry_bytes: int = 4) -> int:
    """Shared memory of one tile: one table of 2^mu entries per base, batch
    row and sub-vector of the K tile, plus a partial sum per row, base and
    batch row."""
    tables = Kb * batch * (Ktile // mu) * (1 << mu) * entry_bytes
    accum = Mtile * Kb * batch * 4
    return tables + accum


def effective_tflops(M: int, N: int, n_sal: int, B: int, seconds: float) -> float:
    """Equivalent fp16 work 2*M*(N + N_sal)*B per second, in TFLOP/s."""
    return 2.0 * M * (N + n_sal) * B / seconds / 1e12

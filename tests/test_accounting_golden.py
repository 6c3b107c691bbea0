"""Pins for the storage / shared-memory / throughput accounting against the
figures the pages print (tests/golden/pages_figures.json, each cited), and
for the naive layout packer against its own inverse."""
import json
import os

import numpy as np
import pytest

from oracle import accounting, layout

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_figures.json")))


def test_smem_footprint_mu8_is_136_kib():
    g = GOLDEN["smem_mu8"]
    p = g["params"]
    b = accounting.lut_smem_bytes(p["Kb"], p["batch"], p["Ktile"], p["mu"], p["Mtile"])
    assert b == g["value_kib"] * 1024


def test_smem_footprint_mu4_at_most_24_kib():
    g = GOLDEN["smem_mu4"]
    p = g["params"]
    b = accounting.lut_smem_bytes(p["Kb"], p["batch"], p["Ktile"], p["mu"], p["Mtile"])
    assert b <= g["max_kib"] * 1024
    # halving mu shrinks the tables 2^8/8 -> 2^4/4 per column: 8x fewer table bytes
    b8 = accounting.lut_smem_bytes(p["Kb"], p["batch"], p["Ktile"], 8, p["Mtile"])
    acc = p["Mtile"] * p["Kb"] * p["batch"] * 4
    assert (b8 - acc) == 8 * (b - acc)


@pytest.mark.parametrize("case", GOLDEN["abw"], ids=lambda c: f"G{c['G']}_s{c['s']}")
def test_average_bit_width(case):
    lead = accounting.abw_leading(case["Kb"], case["Ks"], case["G"], case["s"])
    assert abs(lead - case["bits"]) <= 0.005 + 1e-12
    # every stored item counted, at the 4096 x 4096 shape: within 0.01 bit
    exact = accounting.abw_exact(4096, 4096, case["Kb"], case["Ks"], case["G"], case["s"])
    assert abs(exact - case["bits"]) < 0.015
    if "salient_ratio" in case:
        assert case["s"] / case["G"] == case["salient_ratio"]


def test_effective_tflops_matches_latency():
    g = GOLDEN["kernel_latency"]
    t = accounting.effective_tflops(g["M"], g["N"], 0, g["B"], g["latency_us"] * 1e-6)
    assert abs(t - g["tflops"]) / g["tflops"] < 0.02


def test_lut_example_table_sizes():
    g = GOLDEN["lut_example"]
    from oracle import lut_table, lut_table_sym
    v = np.arange(1, g["activation_len"] + 1, dtype=np.float64)
    assert lut_table(v, g["activation_len"]).size == g["entries"]
    assert lut_table_sym(v, g["activation_len"]).size == g["sym_entries"]


@pytest.mark.parametrize("nb,mu", [(1, 4), (1, 8), (2, 4), (2, 8), (4, 8)])
def test_naive_layout_round_trip(nb, mu):
    rng = np.random.default_rng(nb * 10 + mu)
    M, ncols = 70, 300
    signs = (rng.integers(0, 2, size=(nb, M, ncols)) * 2 - 1).astype(np.int8)
    words = layout.pack_branch(signs, mu)
    assert words.size == layout.branch_words(M, ncols, nb, mu)
    assert np.array_equal(layout.unpack_branch(words, M, ncols, nb, mu), signs)
    # one set bit per +1 sign, none for padding
    assert int(np.unpackbits(words.view(np.uint8)).sum()) == int((signs > 0).sum())

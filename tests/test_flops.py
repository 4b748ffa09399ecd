"""The FLOP accounting reproduces the numbers printed in SequenceO1 App. G.7.

This pins the counting convention (App. G.1: 2mrp per GEMM) and the SA term
4 L_s L d (App. G.3) that the bench uses for its algorithmic TFLOP/s.
"""
import json
import os

import pytest

from sketch_attention_flashsa_b200 import flops

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "flop_model.json")


def _load():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("section", ["printed", "derived_not_printed"])
def test_paper_numbers(section):
    got = flops.paper_numbers()
    for key, ent in _load()[section].items():
        assert round(got[key], ent["digits"]) == pytest.approx(ent["value"], abs=10 ** -ent["digits"] / 2 + 1e-12), key


def test_closed_forms_match_term_lists():
    # App. G.2: N(12 L D^2 + 4 L D h + 20 D^2); App. G.3: N(2 L d^2 + 14 L_s d^2 + 4 L_s L d)
    L, D, h, N = 12345.0, 256.0, 4.0, 3.0
    assert flops.stca(L, N, D, h) == pytest.approx(N * (12 * L * D**2 + 4 * L * D * h + 20 * D**2))
    Ls, d = 96.0, 64.0
    assert flops.sa(L, N, Ls, d) == pytest.approx(N * (2 * L * d**2 + 14 * Ls * d**2 + 4 * Ls * L * d))


def test_hot_path_term_is_affinity_plus_aggregation():
    # the fused kernel's share of one SA layer is exactly the 4 L_s L d term
    L, Ls, d = 1000.0, 512.0, 128.0
    fused = flops.gemm(Ls, d, L) + flops.gemm(Ls, L, d)
    assert flops.sa_forward_flops(int(L), 1, int(Ls), int(d)) == pytest.approx(fused)

"""Measurement arithmetic against the figures the pages print (tests/golden)."""
import json
import os

import pytest

from tiled_exact_attention_fa_b200 import accounting

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_arithmetic.json")
UNITS = {"elements": 1, "Mi-elements": 2**20, "M-elements": 1e6, "MiB": 2**20, "GiB": 2**30,
         "MB": 1e6, "FLOP/byte": 1}
CASES = json.load(open(GOLDEN))["cases"]


@pytest.mark.parametrize("case", CASES, ids=[c["id"] for c in CASES])
def test_page_figure(case):
    got = getattr(accounting, case["quantity"])(**case["args"]) / UNITS[case["unit"]]
    want = case["value"]
    assert abs(got - want) <= case["rel_tol"] * abs(want), (case["cite"], got, want)


def test_headline_flops_and_bytes():
    # bf16 B=2 H=32 N=8192 d=128 causal: 4*B*H*N^2*d / 2
    assert accounting.attention_flops(2, 32, 8192, 128, True) == 2 * 2 * 32 * 8192**2 * 128
    assert accounting.algorithmic_bytes(2, 32, 8192, 128, 2) == 4 * 2 * 32 * 8192 * 128 * 2 + 2 * 32 * 8192 * 4


def test_fp8_bytes():
    # E4M3 B=2 H=32 N=8192 d=128: one-byte Q, K, V, bf16 O, fp32 lse
    rows = 2 * 32 * 8192
    assert accounting.algorithmic_bytes(2, 32, 8192, 128, 1, out_elem_bytes=2) == \
        3 * rows * 128 + 2 * rows * 128 + 4 * rows == 337641472


def test_roofline_min():
    assert accounting.roofline_flops(4, 989e12, 3.35e12) == 4 * 3.35e12
    assert accounting.roofline_flops(1000, 989e12, 3.35e12) == 989e12

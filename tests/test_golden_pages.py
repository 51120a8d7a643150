"""The workload recipe and the work accounting against numbers the pages print
(tests/golden/pages_facts.json, each with its citation). CPU only."""
import json
import os

import pytest

import synth
from group_rational_kan_b200 import accounting

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_facts.json")))


@pytest.mark.parametrize("name", ["kat_t", "kat_s", "kat_b"])
def test_kat_workloads_use_the_pages_group_config(name):
    w = synth.workload(name)
    g = GOLD["group_config"]
    assert w.n_g == g["groups"]
    assert w.m + 1 == g["numerator_coefficients"]
    assert w.n == g["denominator_coefficients"]


def test_forward_flop_formula():
    assert GOLD["extra_flops_formula"]["per_input"] == "2m+2n+3"
    assert accounting.forward_flops_per_element(5, 4) == 2 * 5 + 2 * 4 + 3 == 21


def test_block_accumulation_factor():
    f = GOLD["block_accumulation"]
    r = accounting.flashkat_access_reduction(f["S_block"], f["d_g"])
    assert r == 98304 and abs(r - 98000) / 98000 < 0.01


def test_forward_backward_ratio_units():
    t = GOLD["forward_backward_times_H200"]
    assert abs(t["backward_s"] * 1e3 / t["forward_ms"] - t["stated_ratio"]) < 0.1


def test_bytes_per_element():
    assert accounting.bytes_per_element("step", 1) == 10
    assert accounting.bytes_per_element("step", 0) == 20
    assert accounting.bytes_per_element("backward", 1) == 6
    # one KAT-B step moves 3.0985 GB
    w = synth.workload("kat_b")
    assert abs(w.elems * accounting.bytes_per_element("step", w.dtype) / 1e9 - 3.0985) < 1e-3


def test_backward_flop_count_is_consistent():
    # at (5, 4): powers 4, P 10 + P' 8 + Q 7 + Q' 6, D/r 2, y t nu 3, dx 3, sums 11 + 8
    assert accounting.backward_flops_per_element(5, 4) == 62
    assert accounting.backward_flops_per_element(0, 0) >= 1

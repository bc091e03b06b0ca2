"""Fixtures from tests/golden/: numbers the nanochat pages print, checked
against the one-dial arithmetic (oracle.dims, oracle.param_layout).  The
printed parameter counts are multi-head counts; expanding the shared KV head
of our layout to one per query head must reproduce them to the pages'
rounding, which pins the width rule, the MLP ratio, the untied embeddings and
the vocab of 65,536 together."""
import json
import os

import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_printed_sizes.json")


def _mha_count(depth, vocab=65536):
    D = oracle.dims(depth, vocab)
    C = D["C"]
    n = 0
    for name, rows, cols in oracle.param_layout(depth, vocab):
        if name.endswith(".wk") or name.endswith(".wv"):
            rows = C  # one KV head per query head instead of one shared head
        n += rows * cols
    return n


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"])
def test_printed_sizes(case):
    D = oracle.dims(case["depth"], 65536)
    assert D["C"] == case["width"] and D["H"] == case["heads"] and D["d"] == case["head_dim"]
    n = _mha_count(case["depth"])
    # the pages print three significant digits
    assert abs(n - case["params_approx"]) <= 0.005 * case["params_approx"], (n, case["printed"])


def test_mqa_is_smaller_by_the_kv_heads():
    for depth in (20, 32):
        C = oracle.dims(depth, 65536)["C"]
        mqa = sum(r * c for _, r, c in oracle.param_layout(depth, 65536))
        assert _mha_count(depth) - mqa == depth * 2 * (C - 128) * C

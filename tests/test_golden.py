"""The oracle against its stored regression record (tests/golden/).

The record is written by tests/golden/make_golden.py, which calls only the
oracle; the oracle itself is pinned to the pages and the mathematics in
test_oracle.py.  This test keeps the oracle's arithmetic from changing by
accident.
"""
import json
import os

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "oracle_small_cases.json")
with open(GOLDEN) as f:
    CASES = json.load(f)


@pytest.mark.parametrize("name", sorted(CASES))
def test_oracle_reproduces_golden(name):
    case = CASES[name]
    w = workloads.make_workload(**case["args"])
    exp = case["expected"]
    if case["extra"]:
        r = oracle.block_attn(w, case["extra"]["block_size"], case["extra"]["top_blocks"])
        assert r["block_idx"].ravel().tolist() == exp["block_idx"]
    else:
        r = oracle.topk_attn(w, case["k"])
        assert r["idx"].ravel().tolist() == exp["idx"]
        np.testing.assert_allclose(r["tail"].ravel(), exp["tail"], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(r["out"][..., :16].ravel(), exp["out16"], rtol=1e-12, atol=1e-15)

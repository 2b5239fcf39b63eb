"""Parity at the workloads' full sizes, in the configuration bench.py times
(normalise the raw corpus and queries on the GPU, then score), against the
fp64 oracle: every query for the smaller workloads, a seeded sample of 16
queries for the two largest (the oracle sorts all 20-50 million scores of
each sampled query). GPU; several minutes and tens of GB of host memory.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
import workloads as W

pytestmark = pytest.mark.gpu

tt = pytest.importorskip("exact_inner_product_b200")


@pytest.mark.parametrize("name", ["tiny_f32", "stream_b1", "small_batch", "large_batch", "masked_fused"])
def test_full_size_parity(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    oracle.set_threads(oracle.max_threads())
    w = W.workload(name)
    res, st = parity.run_case(w)
    expect_path = 1 if (w.store == "f32" or w.b <= 8) else 2 if (w.b < 256 or w.store == "raw") else 3
    assert st["path"] == expect_path
    assert res["queries"] == len(W.oracle_query_ids(w))
    assert res["max_abs_err"] <= w.tolerance
    # members of the true top-k that no rounding can displace were all returned
    assert res["sure_checked"] > 0, res
    torch.cuda.empty_cache()

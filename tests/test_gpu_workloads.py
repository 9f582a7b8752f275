"""The five named workloads at full size, in the launch configuration the
benchmark times (one sage_attn_fwd call on the default stream).

Pre-pass outputs are compared bit for bit over the whole tensors; the output
is compared on sampled query tiles (first, last/ragged and random ones) that
the oracle computes row by row.  Against the mirror: max |diff| <= 2e-2 and
cosine >= 0.9999.  Against exact fp64 attention: relative L1 <= 0.06 and
cosine >= 0.998, except the workload whose Q/K/V carry x20 channel outliers,
where per-block INT8 scales of Q and K are dominated by the outlier channels
and the method itself (the oracle's mirror, not only the GPU) sits near 0.04
relative L1 / 0.996 cosine; there the bound is relative L1 <= 0.06 and
cosine >= 0.99.
"""
import json
import os

import pytest

from quantized_attention_subtract_b200.workloads import WORKLOADS

from _common import (EXACT_COS, EXACT_REL_L1, MIRROR_COS, MIRROR_MAX_ABS, assert_prepass_bit_exact,
                     compare_output, run_both, sample_tiles)

pytestmark = pytest.mark.gpu

RUNS = [(name, None) for name in WORKLOADS] + [("gqa_cross_nq2048_nkv8192_d96_fp16", False)]


@pytest.mark.parametrize("name,smooth_k", RUNS, ids=[f"{n}-sk{s}" for n, s in RUNS])
def test_workload_full_size(name, smooth_k):
    w = WORKLOADS[name]
    if smooth_k is not None:
        w = w.with_(smooth_k=smooth_k)
    q, k, v, pr, pre, g = run_both(w)
    assert_prepass_bit_exact(w, pre, g)
    tiles = sample_tiles(pr, 6, seed=1)
    r = compare_output(pr, pre, q, k, v, g, tiles)
    report = os.environ.get("SAGE_TEST_REPORT")
    if report:
        with open(report, "a") as f:
            f.write(json.dumps(dict(workload=name, smooth_k=w.smooth_k, **r)) + "\n")
    assert r["max_abs"] <= MIRROR_MAX_ABS and r["cos"] >= MIRROR_COS, r
    if w.outlier_channels:
        assert r["rel_l1_exact"] <= 0.06 and r["cos_exact"] >= 0.99, r
    else:
        assert r["rel_l1_exact"] <= EXACT_REL_L1 and r["cos_exact"] >= EXACT_COS, r

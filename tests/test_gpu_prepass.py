"""GPU pre-pass vs the oracle, bit for bit: INT8 codes and scales of Q and K,
FP8 codes and scales of V, the K / V / per-block Q means, and zero padding."""
import pytest

from quantized_attention_subtract_b200.workloads import random_problem

from _common import assert_prepass_bit_exact, run_both

pytestmark = pytest.mark.gpu

CASES = [
    dict(args=(1, 2, 2, 256, 256, 64), dtype="fp16"),
    dict(args=(2, 4, 2, 300, 200, 96), dtype="bf16", layout="NHD"),
    dict(args=(1, 8, 1, 130, 1000, 128), dtype="bf16"),
    dict(args=(2, 3, 3, 129, 65, 64), dtype="fp16", smooth_k=False),
    dict(args=(1, 4, 2, 384, 700, 128), dtype="fp16", smooth_q=True, smooth_v=True),
    dict(args=(1, 2, 1, 1, 1, 96), dtype="bf16", smooth_v=True),
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_prepass_bit_exact(case):
    flags = {k: v for k, v in case.items() if k in ("smooth_k", "smooth_q", "smooth_v", "is_causal")}
    w = random_problem(*case["args"], layout=case.get("layout", "HND"), dtype=case["dtype"],
                       seed=7, k_offset_sigma=5.0, **flags)
    q, k, v, pr, pre, g = run_both(w)
    assert_prepass_bit_exact(w, pre, g)


def test_delta_s_matches_oracle():
    import numpy as np
    import oracle
    w = random_problem(1, 4, 2, 300, 500, 128, dtype="bf16", seed=3, smooth_q=True)
    q, k, v, pr, pre, g = run_both(w)
    K2 = np.float32(pr.resolved_sm_scale()) * np.float32(1.4426950408889634)
    dsk = g.views["dsk"].cpu().numpy()
    for b, h, qt in [(0, 0, 0), (0, 3, 2), (0, 1, 1)]:
        want = oracle.delta_s(pr, pre, b, h, qt) * float(K2)
        got = dsk[b, h, qt, : pr.Nkv]
        assert np.max(np.abs(got - want)) <= 1e-5 * np.max(np.abs(want)) + 1e-6

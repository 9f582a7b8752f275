"""The 4-bit Q/K variant on the GPU (qk_bits = 4: INT4 codes in [-7, 7] on
the 8-bit path's blocks, multiplied exactly on the INT8 tensor path;
"SageAttention2: Technical report", sections 1 and 3), through the C ABI,
against the oracle run with the same setting.

- Pre-pass outputs bit for bit (codes, scales, means); the FP8 V codes equal
  the 8-bit run's.
- S tiles the production kernel reads from tensor memory equal int64 dot
  products of the INT4 codes.
- Outputs against the oracle's mirror: max |diff| beyond the ambiguous-FP8
  band and half an output ulp <= 2e-2, cosine >= 0.9999; against exact fp64
  attention no worse than the oracle's own 4-bit error + 0.002.
- The public entry points (batched, variable-length, host tensors) take the
  switch and give the params path's result bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_attention_subtract_b200 import binding, sageattn, sageattn_varlen
from quantized_attention_subtract_b200.workloads import generate, generate_varlen, random_problem

from _common import (MIRROR_COS, MIRROR_MAX_ABS, DeviceRun, assert_prepass_bit_exact, compare_output,
                     half_ulp, oracle_problem, run_both)

pytestmark = pytest.mark.gpu

CASES = [
    dict(args=(1, 2, 2, 256, 300, 64), dtype="fp16"),
    dict(args=(2, 4, 2, 300, 200, 96), dtype="bf16", layout="NHD", smooth_q=True, smooth_v=True),
    dict(args=(1, 4, 1, 640, 640, 128), dtype="bf16", is_causal=True),
    dict(args=(1, 8, 2, 129, 1100, 128), dtype="fp16", smooth_q=True),
    dict(args=(2, 3, 3, 390, 260, 64), dtype="bf16", layout="NHD", is_causal=True, smooth_k=False),
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_int4_attention_matches_oracle(case):
    flags = {k: v for k, v in case.items() if k in ("smooth_k", "smooth_q", "smooth_v", "is_causal")}
    w = random_problem(*case["args"], layout=case.get("layout", "HND"), dtype=case["dtype"],
                       seed=17, k_offset_sigma=5.0, qk_bits=4, **flags)
    q, k, v, pr, pre, g = run_both(w)
    assert_prepass_bit_exact(w, pre, g)
    assert int(g.views["q8"].abs().max()) == 7 and int(g.views["k8"].abs().max()) == 7
    r = compare_output(pr, pre, q, k, v, g, oracle.all_tiles(pr))
    assert r["max_abs_excess"] <= MIRROR_MAX_ABS and r["cos"] >= MIRROR_COS, r
    assert r["rel_l1_exact"] <= r["mirror_rel_l1_exact"] + 0.002, r
    # the V path is the 8-bit run's
    g8 = DeviceRun(w.with_(qk_bits=8), q, k, v, run_attention=False)
    assert torch.equal(g.views["v8t"], g8.views["v8t"]) and torch.equal(g.views["v_scale"], g8.views["v_scale"])


@pytest.mark.parametrize("D,causal", [(64, False), (128, True)])
def test_int4_s_tiles_bit_exact(D, causal):
    w = random_problem(1, 4, 2, 384, 384, D, dtype="bf16", seed=D + 1, is_causal=causal, qk_bits=4)
    q, k, v = generate(w)
    pre = oracle.prepass(oracle_problem(w), q, k, v)
    g = DeviceRun(w, q, k, v, run_attention=False)
    for b, h, qt, kt in [(0, 0, 0, 0), (0, 3, 2, 2), (0, 1, 2, 0), (0, 2, 1, 1)]:
        s = binding.debug_dump_s(g.p, b, h, qt, kt, "cuda").cpu().numpy().astype(np.int64)
        torch.cuda.synchronize()
        assert binding.device_status(g.p) == 0
        qb = pre["q8"][b, h, qt * 128: qt * 128 + 128].astype(np.int64)
        kb = pre["k8"][b, h // 2, kt * 128: kt * 128 + 128].astype(np.int64)
        assert np.array_equal(s, qb @ kb.T), (b, h, qt, kt)


def test_int4_public_api_and_host_tensors():
    w = random_problem(1, 4, 2, 300, 300, 128, dtype="bf16", seed=3, qk_bits=4)
    q, k, v = generate(w)
    g = DeviceRun(w, q, k, v)
    got = sageattn(g.q, g.k, g.v, "HND", qk_bits=4)
    torch.cuda.synchronize()
    assert torch.equal(got, g.out)
    host = sageattn(g.q.cpu(), g.k.cpu(), g.v.cpu(), "HND", qk_bits=4)
    torch.cuda.synchronize()
    assert torch.equal(host, g.out.cpu())
    # 8 bits on the same inputs is a different result
    assert not torch.equal(sageattn(g.q, g.k, g.v, "HND"), g.out)


def test_int4_varlen_matches_oracle():
    Hq, Hkv, D = 4, 2, 128
    lq, lk = [300, 1, 129, 500], [300, 7, 129, 700]
    cu_q, cu_kv, q, k, v = generate_varlen(Hq, Hkv, D, lq, lk, "bf16", seed=5)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    qd, kd, vd = dev(q), dev(k), dev(v)
    out = sageattn_varlen(qd, kd, vd, cu_q, cu_kv, is_causal=True, qk_bits=4)
    torch.cuda.synchronize()
    r = oracle.varlen_attention(Hq, Hkv, D, cu_q, cu_kv, q, k, v, dtype="bf16", is_causal=True,
                                with_uncertainty=True, qk_bits=4)
    got = out.double().cpu().numpy()
    m, u = r["out"], r["unc"]
    excess = np.max(np.abs(got - m) - u - half_ulp(np.maximum(np.abs(got), np.abs(m)), "bf16"))
    cos = (got * m).sum() / np.linalg.norm(got) / np.linalg.norm(m)
    assert excess <= MIRROR_MAX_ABS and cos >= MIRROR_COS, (excess, cos)

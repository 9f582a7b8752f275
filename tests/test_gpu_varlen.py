"""Variable-length batches on the GPU (packed sequences with offsets), through
the C ABI, against the oracle run once per sequence.

Per configuration: the output against the oracle's mirror (max |diff| beyond
the ambiguous-FP8 band and half an output ulp <= 2e-2, cosine >= 0.9999) and
against exact fp64 attention (relative L1 <= 0.06, cosine >= 0.998); every
sequence's pre-pass outputs bit for bit; and the whole batch bit for bit
against separate calls, one per sequence, of the batched path."""
import numpy as np
import pytest
import torch

import oracle
from quantized_attention_subtract_b200 import binding, sageattn, sageattn_varlen
from quantized_attention_subtract_b200.workloads import generate_varlen

from _common import EXACT_COS, EXACT_REL_L1, MIRROR_COS, MIRROR_MAX_ABS, half_ulp

pytestmark = pytest.mark.gpu

CASES = [
    dict(H=(4, 4), D=128, dtype="bf16", lq=[300, 1, 129, 700], lk=[300, 1, 129, 700], causal=False),
    dict(H=(4, 2), D=64, dtype="fp16", lq=[256, 0, 37, 513], lk=[512, 9, 37, 200], causal=True),
    dict(H=(6, 2), D=96, dtype="bf16", lq=[130, 255, 64], lk=[1000, 2, 300], causal=False,
         smooth_v=True),
    dict(H=(2, 1), D=128, dtype="fp16", lq=[5, 400], lk=[5, 400], causal=True, smooth_q=True),
]


def _dev(bits, dtype):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    return t.view(torch.float16 if dtype == "fp16" else torch.bfloat16)


def _run(case, seed=13):
    Hq, Hkv = case["H"]
    cu_q, cu_kv, q, k, v = generate_varlen(Hq, Hkv, case["D"], case["lq"], case["lk"], case["dtype"],
                                           seed=seed)
    qd, kd, vd = (_dev(x, case["dtype"]) for x in (q, k, v))
    flags = dict(is_causal=case["causal"], smooth_q=case.get("smooth_q", False),
                 smooth_v=case.get("smooth_v", False))
    out = torch.empty_like(qd)
    p = binding.make_varlen_params(qd, kd, vd, out, cu_q, cu_kv, **flags)
    ws = binding.alloc_workspace(p, qd.device)
    binding.attn_fwd(p, qd.device)
    torch.cuda.synchronize()
    assert binding.device_status(p) == 0
    return cu_q, cu_kv, q, k, v, (qd, kd, vd), out, p, ws, flags


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_varlen_matches_oracle(case):
    Hq, Hkv = case["H"]
    cu_q, cu_kv, q, k, v, _, out, p, ws, flags = _run(case)
    r = oracle.varlen_attention(Hq, Hkv, case["D"], cu_q, cu_kv, q, k, v, dtype=case["dtype"],
                                with_uncertainty=True, exact=True, **flags)
    got = out.double().cpu().numpy()
    m, u, e = r["out"], r["unc"], r["exact"]
    d = np.abs(got - m)
    excess = np.max(d - u - half_ulp(np.maximum(np.abs(got), np.abs(m)), case["dtype"]))
    cos = (got * m).sum() / np.linalg.norm(got) / np.linalg.norm(m)
    assert excess <= MIRROR_MAX_ABS and cos >= MIRROR_COS, (excess, cos)
    rel = np.abs(got - e).sum() / np.abs(e).sum()
    cos_e = (got * e).sum() / np.linalg.norm(got) / np.linalg.norm(e)
    assert rel <= EXACT_REL_L1 and cos_e >= EXACT_COS, (rel, cos_e)
    # per-sequence pre-pass outputs, bit for bit
    V = {n: (t.cpu().numpy() if isinstance(t, torch.Tensor) else t)
         for n, t in binding.workspace_views(p, ws).items()}
    D = case["D"]
    for b, pre in enumerate(r["pre"]):
        if pre is None:
            continue
        lq, lk = case["lq"][b], case["lk"][b]
        assert np.array_equal(V["q8"][b, :, :lq, :D], pre["q8"][0]), ("q8", b)
        assert np.array_equal(V["k8"][b, :, :lk, :D], pre["k8"][0]), ("k8", b)
        assert np.array_equal(V["v8t"][b].transpose(0, 2, 1)[:, :lk], pre["v8"][0]), ("v8", b)
        assert np.array_equal(V["q_scale"][b, :, :pre["q_scale"].shape[-1]], pre["q_scale"][0]), b
        assert np.array_equal(V["k_scale"][b, :, :pre["k_scale"].shape[-1]], pre["k_scale"][0]), b
        assert np.array_equal(V["v_scale"][b], pre["v_scale"][0]), ("v_scale", b)


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_varlen_equals_one_call_per_sequence(case):
    cu_q, cu_kv, q, k, v, (qd, kd, vd), out, p, ws, flags = _run(case, seed=17)
    for b in range(len(case["lq"])):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_kv[b]), int(cu_kv[b + 1])
        if q1 == q0:
            continue
        ref = sageattn(qd[q0:q1][None], kd[k0:k1][None], vd[k0:k1][None], tensor_layout="NHD",
                       **flags)
        torch.cuda.synchronize()
        assert torch.equal(out[q0:q1], ref[0]), b


def test_public_varlen_call_matches_params_path():
    case = CASES[1]
    cu_q, cu_kv, q, k, v, (qd, kd, vd), out, p, ws, flags = _run(case, seed=19)
    a = sageattn_varlen(qd, kd, vd, torch.from_numpy(cu_q), torch.from_numpy(cu_kv), **flags)
    torch.cuda.synchronize()
    assert torch.equal(a, out)

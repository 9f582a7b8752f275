"""GPU attention vs the oracle (the plain online softmax of the quantised
method): max |diff| <= 2e-2 beyond the effect of FP8 codes of P that fp32
rounding leaves ambiguous and half an ulp of the 16-bit output, cosine >=
0.9999; and vs exact fp64 attention (relative L1 <= 0.06, cosine >= 0.998).
Every query tile of small problems spanning several tiles and query-tile
pairs, ragged tails, a missing second tile of a pair, both layouts, GQA,
causal masking, all head dims and flags, plus the degenerate shapes."""
import numpy as np
import pytest
import torch

import oracle
from quantized_attention_subtract_b200 import binding, sageattn
from quantized_attention_subtract_b200.workloads import generate, random_problem

from _common import (EXACT_COS, EXACT_REL_L1, MIRROR_COS, MIRROR_MAX_ABS, DeviceRun,
                     assert_prepass_bit_exact, compare_output, oracle_problem, run_both, to_device)

pytestmark = pytest.mark.gpu

CASES = [
    dict(args=(1, 2, 2, 256, 256, 64), dtype="fp16"),                       # the 256 / d64 case
    dict(args=(2, 4, 2, 300, 200, 96), dtype="bf16", layout="NHD"),
    dict(args=(1, 4, 1, 384, 384, 128), dtype="bf16", is_causal=True),
    dict(args=(1, 4, 4, 200, 520, 64), dtype="fp16", is_causal=True),       # causal, Nq != Nkv
    dict(args=(2, 2, 2, 260, 260, 96), dtype="bf16", layout="NHD", is_causal=True),
    dict(args=(1, 2, 2, 256, 512, 64), dtype="fp16", smooth_k=False),
    dict(args=(1, 4, 2, 256, 640, 128), dtype="fp16", smooth_q=True, smooth_v=True),
    dict(args=(1, 8, 1, 129, 1100, 128), dtype="bf16"),                     # GQA 8:1, ragged
    dict(args=(1, 2, 2, 1, 1, 64), dtype="fp16"),                           # one query, one key
    dict(args=(1, 2, 1, 5, 3000, 96), dtype="fp16", smooth_v=True),
    # NHD without smooth_k (the pre-pass reads K only for quantisation) and
    # NHD with smoothed Q and V, both through the pre-pass's tensor maps
    dict(args=(2, 4, 2, 200, 333, 128), dtype="bf16", layout="NHD", smooth_k=False),
    dict(args=(1, 4, 4, 260, 390, 96), dtype="fp16", layout="NHD", smooth_q=True, smooth_v=True),
    # five query tiles: the last pair has no second tile; causal, the first
    # tile of a pair stops one KV tile before the second
    dict(args=(1, 2, 2, 640, 700, 128), dtype="bf16", is_causal=True),
    dict(args=(2, 3, 1, 520, 900, 64), dtype="fp16"),
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_attention_matches_oracle(case):
    flags = {k: v for k, v in case.items() if k in ("smooth_k", "smooth_q", "smooth_v", "is_causal")}
    w = random_problem(*case["args"], layout=case.get("layout", "HND"), dtype=case["dtype"],
                       seed=11, k_offset_sigma=5.0, **flags)
    q, k, v, pr, pre, g = run_both(w)
    assert_prepass_bit_exact(w, pre, g)
    r = compare_output(pr, pre, q, k, v, g, oracle.all_tiles(pr))
    assert r["max_abs_excess"] <= MIRROR_MAX_ABS and r["cos"] >= MIRROR_COS, r
    assert r["rel_l1_exact"] <= EXACT_REL_L1 and r["cos_exact"] >= EXACT_COS, r


HALVES = [
    dict(args=(2, 4, 2, 300, 520, 128), dtype="bf16", layout="HND"),
    dict(args=(1, 4, 4, 200, 520, 96), dtype="fp16", layout="NHD", is_causal=True),
    dict(args=(1, 2, 2, 129, 300, 64), dtype="bf16", layout="NHD"),
]


@pytest.mark.parametrize("case", HALVES, ids=[str(i) for i in range(len(HALVES))])
def test_whole_pass_equals_its_two_halves(case):
    """sage_attn_fwd and sage_quantize followed by sage_attn_quantized on the
    same inputs give bit-identical outputs and workspace contents."""
    flags = {k: v for k, v in case.items() if k == "is_causal"}
    w = random_problem(*case["args"], layout=case["layout"], dtype=case["dtype"], seed=21, **flags)
    q, k, v = generate(w)
    whole = DeviceRun(w, q, k, v)
    sep = DeviceRun(w, q, k, v, run_attention=False)
    binding.attn_quantized(sep.p, sep.q.device)
    torch.cuda.synchronize()
    assert binding.device_status(sep.p) == 0
    assert torch.equal(whole.out, sep.out)
    for name in ("q8", "q_scale", "k8", "k_scale", "v8t", "v_scale"):
        assert torch.equal(whole.views[name], sep.views[name]), name


def test_public_api_matches_params_path_and_host_tensors():
    w = random_problem(1, 4, 2, 300, 300, 128, dtype="bf16", seed=2)
    q, k, v = generate(w)
    g = DeviceRun(w, q, k, v)
    a = sageattn(g.q, g.k, g.v, tensor_layout="HND", is_causal=False)
    torch.cuda.synchronize()
    assert torch.equal(a, g.out)
    h = sageattn(g.q.cpu().pin_memory(), g.k.cpu().pin_memory(), g.v.cpu().pin_memory())
    torch.cuda.synchronize()
    assert torch.equal(h, g.out.cpu())


def test_host_tensors_nhd():
    """Host tensors in NHD layout (copied one whole batch entry at a time) give
    the device path's output bit for bit."""
    w = random_problem(2, 4, 2, 300, 260, 64, layout="NHD", dtype="fp16", seed=6)
    q, k, v = generate(w)
    g = DeviceRun(w, q, k, v)
    h = sageattn(g.q.cpu().pin_memory(), g.k.cpu().pin_memory(), g.v.cpu().pin_memory(),
                 tensor_layout="NHD")
    torch.cuda.synchronize()
    assert torch.equal(h, g.out.cpu())


def test_strided_inputs():
    """q, k, v as views with padded token strides (still 16-byte aligned rows)."""
    w = random_problem(1, 2, 2, 256, 256, 64, dtype="fp16", seed=5)
    q, k, v = generate(w)
    dense = DeviceRun(w, q, k, v)
    big = torch.zeros(1, 2, 256, 128, dtype=torch.float16, device="cuda")
    views = []
    for t in (dense.q, dense.k, dense.v):
        b = big.clone()
        b[..., :64] = t
        views.append(b[..., :64])
    out = sageattn(*views)
    torch.cuda.synchronize()
    assert torch.equal(out, dense.out)


def test_empty_queries_is_a_no_op():
    q = torch.zeros(1, 2, 0, 64, dtype=torch.float16, device="cuda")
    k = torch.zeros(1, 2, 10, 64, dtype=torch.float16, device="cuda")
    out = sageattn(q, k, k)
    assert out.shape == q.shape


def test_no_keys_is_rejected():
    q = torch.zeros(1, 2, 4, 64, dtype=torch.float16, device="cuda")
    k = torch.zeros(1, 2, 0, 64, dtype=torch.float16, device="cuda")
    with pytest.raises(binding.SageError):
        sageattn(q, k, k)


def test_constant_v_rows_give_the_constant():
    w = random_problem(1, 2, 2, 256, 700, 128, dtype="bf16", seed=4)
    q, k, v = generate(w)
    const = np.linspace(-2, 2, 128, dtype=np.float32)
    import torch as _t
    vb = _t.from_numpy(np.broadcast_to(const, (1, 2, 700, 128)).copy()).to(_t.bfloat16)
    v = vb.view(_t.int16).numpy().view(np.uint16)
    g = DeviceRun(w, q, k, v)
    c = vb[0, 0, 0].double().numpy()
    o = g.out_f64()
    assert np.all(np.abs(o - c) <= 2.0 ** -4 * np.abs(c) + 2 ** -8)

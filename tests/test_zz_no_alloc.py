"""sage_attn_fwd_noalloc: the entry point for callers that cannot allocate
device memory (hosts with a fixed, pre-planned memory budget, or latency-
critical loops where cudaMalloc would synchronise the device).  It uses the
library's static 64 MiB scratch instead of a caller workspace.

Checked through the C ABI against sage_attn_fwd on the same inputs.  Both run
the same kernels on the same inputs, so the outputs must be bit-identical.
The calls come in a sequence that changes shape on the one shared array
(large D = 128, then a ragged D = 96, then causal D = 64, 4-bit Q/K codes,
then back), so stale padding, scales or accumulators left by a larger earlier
call would show;
variable-length batches (sequence offsets and running totals in the scratch)
and smoothed Q and V (the per-block means and the dS rows) are covered too.
The device status the no-alloc path leaves is read back through its own
query.  The size limit is enforced before anything runs.  This file sorts
last so that a run stopping at the first failure has run every other test
first; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from quantized_attention_subtract_b200 import binding
from quantized_attention_subtract_b200.workloads import generate, generate_varlen, random_problem

from _common import to_device

pytestmark = pytest.mark.gpu

SEQUENCE = [
    ((2, 4, 2, 900, 1400, 128), dict(dtype="bf16")),
    ((1, 6, 3, 260, 261, 96), dict(dtype="fp16", layout="NHD")),
    ((1, 4, 1, 300, 300, 64), dict(dtype="bf16", is_causal=True)),
    ((1, 4, 2, 256, 640, 128), dict(dtype="fp16", smooth_q=True, smooth_v=True)),
    ((1, 4, 2, 300, 500, 128), dict(dtype="bf16", qk_bits=4)),
    ((2, 4, 2, 900, 1400, 128), dict(dtype="bf16")),
]


def _pair(args, kw, seed):
    flags = {k: v for k, v in kw.items() if k in ("is_causal", "smooth_q", "smooth_v")}
    w = random_problem(*args, layout=kw.get("layout", "HND"), dtype=kw["dtype"], seed=seed, **flags)
    q, k, v = (to_device(x, w.dtype) for x in generate(w, seed))
    fl = dict(smooth_q=w.smooth_q, smooth_v=w.smooth_v, qk_bits=kw.get("qk_bits", 8))
    ref = torch.empty_like(q)
    p = binding.make_params(q, k, v, ref, w.layout, w.is_causal, None, True, **fl)
    ws = binding.alloc_workspace(p, q.device)
    binding.attn_fwd(p, q.device)
    got = torch.empty_like(q)
    pn = binding.make_params(q, k, v, got, w.layout, w.is_causal, None, True, **fl)
    binding.attn_fwd_noalloc(pn, q.device)
    torch.cuda.synchronize()
    assert binding.device_status(p) == 0
    assert binding.noalloc_device_status(pn, q.device) == 0
    del ws
    return got, ref


def test_noalloc_matches_workspace_path_across_shape_changes():
    """Two rounds of the shape-changing sequence (each call with its own
    inputs): every no-alloc output equals the workspace path's bit for bit."""
    for rnd in range(2):
        for n, (args, kw) in enumerate(SEQUENCE):
            got, ref = _pair(args, kw, seed=31 + 10 * rnd + n)
            assert torch.equal(got, ref), (rnd, n, args, kw)


def test_noalloc_variable_length_batch():
    """A packed batch after a larger batched call: the sequence offsets and
    running unit totals in the scratch are rewritten by each call."""
    _pair(*SEQUENCE[0], seed=41)
    rng = np.random.default_rng(5)
    for seed in (42, 43):
        lq = rng.integers(1, 700, 5)
        lk = rng.integers(1, 900, 5)
        cu_q, cu_kv, q, k, v = generate_varlen(4, 2, 128, lq, lk, "bf16", seed=seed)
        qd, kd, vd = (to_device(x, "bf16") for x in (q, k, v))
        ref, got = torch.empty_like(qd), torch.empty_like(qd)
        p = binding.make_varlen_params(qd, kd, vd, ref, cu_q, cu_kv)
        ws = binding.alloc_workspace(p, qd.device)
        binding.attn_fwd(p, qd.device)
        pn = binding.make_varlen_params(qd, kd, vd, got, cu_q, cu_kv)
        binding.attn_fwd_noalloc(pn, qd.device)
        torch.cuda.synchronize()
        assert binding.noalloc_device_status(pn, qd.device) == 0
        assert torch.equal(got, ref), seed
        del ws


def test_noalloc_rejects_problems_over_the_limit():
    p = binding.Params()
    p.B, p.Hq, p.Hkv, p.Nq, p.Nkv, p.D = 4, 32, 32, 4096, 4096, 128
    assert binding.workspace_bytes(p) > binding.NOALLOC_MAX_WORKSPACE_BYTES
    q = torch.zeros(1, dtype=torch.float16, device="cuda")
    p.q = p.k = p.v = p.out = q.data_ptr()
    for name in ("q_strides", "k_strides", "v_strides", "o_strides"):
        getattr(p, name)[:] = [32 * 4096 * 128, 4096 * 128, 128, 1]
    code = binding.lib().sage_attn_fwd_noalloc(ctypes.byref(p), None)
    assert code == 6  # SAGE_ERR_WORKSPACE, nothing enqueued

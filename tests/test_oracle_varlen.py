"""Pins of the variable-length oracle (a batch of packed sequences, each its
own problem; "sageattention" package page, "What it is" / "Use it for")."""
import numpy as np

import oracle
from quantized_attention_subtract_b200.workloads import _to_bits, generate_varlen

LQ, LK = [70, 200, 1, 0, 130], [90, 130, 5, 0, 257]


def test_constant_v_per_sequence_gives_that_sequence_s_constant():
    """With V smoothing and V constant over each sequence's tokens (a
    different constant per sequence), V - mean_v is zero, so every output row
    is exactly its own sequence's constant: a row that saw another sequence's
    keys or values would carry that sequence's constant instead."""
    cu_q, cu_kv, q, k, _ = generate_varlen(2, 1, 64, LQ, LK, "fp16", seed=3)
    rng = np.random.default_rng(7)
    consts = (rng.standard_normal((len(LK), 1, 64)) * 2).astype(np.float16).astype(np.float32)
    vf = np.zeros((int(cu_kv[-1]), 1, 64), np.float32)
    for b in range(len(LK)):
        vf[cu_kv[b]:cu_kv[b + 1]] = consts[b]
    r = oracle.varlen_attention(2, 1, 64, cu_q, cu_kv, q, k, _to_bits(vf, "fp16"), smooth_v=True,
                                is_causal=True)
    for b in range(len(LQ)):
        rows = r["out"][cu_q[b]:cu_q[b + 1]]
        assert np.array_equal(rows, np.broadcast_to(consts[b].astype(np.float64), rows.shape)), b


def test_first_causal_query_of_each_sequence_sees_only_its_first_key():
    """Causal masking is top-left within each sequence: query 0 of sequence b
    attends to key 0 of sequence b alone, so exact attention returns that
    value row exactly, and the quantised mirror returns it within the FP8
    rounding of V (relative 2^-4 of the channel scale)."""
    cu_q, cu_kv, q, k, v = generate_varlen(2, 2, 64, LQ, LK, "bf16", seed=5)
    r = oracle.varlen_attention(2, 2, 64, cu_q, cu_kv, q, k, v, dtype="bf16", is_causal=True,
                                exact=True)
    vd = oracle.to_double(oracle.Problem(1, 2, 2, 1, 1, 64, dtype="bf16"), v)
    for b in range(len(LQ)):
        if LQ[b] == 0:
            continue
        v0 = vd[cu_kv[b]]
        assert np.array_equal(r["exact"][cu_q[b]], v0), b
        vmax = np.abs(vd[cu_kv[b]:cu_kv[b + 1]]).max(axis=0)
        assert np.all(np.abs(r["out"][cu_q[b]] - v0) <= vmax * 2.0 ** -4 + 1e-12), b


def test_sequences_are_independent():
    """Changing one sequence's K and V changes no other sequence's output."""
    cu_q, cu_kv, q, k, v = generate_varlen(2, 1, 64, LQ, LK, "fp16", seed=9)
    a = oracle.varlen_attention(2, 1, 64, cu_q, cu_kv, q, k, v)
    k2, v2 = k.copy(), v.copy()
    s = slice(int(cu_kv[1]), int(cu_kv[2]))
    k2[s] = k2[s][::-1]
    v2[s] = _to_bits(np.full(v2[s].shape, 3.0, np.float32), "fp16")
    b = oracle.varlen_attention(2, 1, 64, cu_q, cu_kv, q, k2, v2)
    other = np.ones(int(cu_q[-1]), bool)
    other[cu_q[1]:cu_q[2]] = False
    assert np.array_equal(a["out"][other], b["out"][other])
    assert not np.array_equal(a["out"][~other], b["out"][~other])

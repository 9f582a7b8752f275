"""Pins of the oracle's 4-bit Q/K variant ("SageAttention2: Technical
report", section 1: Q and K quantised to INT4 at warp level; section 3: the
sensitive layers keep 8 bits, the others take 4).

- The blocks are the 8-bit path's (one scale per query token, one per 32
  keys) with codes in [-7, 7]: scale = amax/7, every nonzero block reaches
  +-7, and the round trip is within half a step (numpy on the decoded inputs).
- Inputs already on a 4-bit grid (a power of two times integers in [-7, 7],
  with +-7 in every block) are quantised without error, so the 4-bit path
  reproduces the unquantised Q K^T path exactly; a scale of amax/8 or
  amax/15, or codes clamped to another range, would not.
- Section 2 of the same report: subtracting the channel mean of Q before
  quantising is what keeps the 4-bit error small when Q has a common channel
  offset; with an offset it cuts the 4-bit error at least in half, without
  one it changes little.
"""
import numpy as np
import pytest

import oracle
from quantized_attention_subtract_b200.workloads import _to_bits, generate, random_problem


def _problem(w, **kw):
    d = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, Nq=w.Nq, Nkv=w.Nkv, D=w.D, layout=w.layout, dtype=w.dtype,
             is_causal=w.is_causal, smooth_k=w.smooth_k, smooth_q=w.smooth_q, smooth_v=w.smooth_v)
    d.update(kw)
    return oracle.Problem(**d)


def _rel_l1(a, b):
    return np.abs(a - b).sum() / np.abs(b).sum()


def _check_blocks(x, codes, scales, blk, n):
    for i in range((n + blk - 1) // blk):
        sl = slice(i * blk, min((i + 1) * blk, n))
        xb, cb, s = x[..., sl, :], codes[..., sl, :].astype(np.float64), scales[..., i]
        amax = np.abs(xb).max(axis=(-2, -1))
        assert np.array_equal(s, amax.astype(np.float32) / np.float32(7))
        assert np.all(np.abs(cb) <= 7)
        nz = s > 0
        assert np.all(np.abs(cb).max(axis=(-2, -1))[nz] == 7)
        err = np.abs(xb - cb * s[..., None, None])
        assert np.all(err <= s[..., None, None] * (0.5 + 2.0 ** -16))


def test_int4_blocks_per_token_and_per_32_keys():
    w = random_problem(2, 4, 2, 300, 200, 64, dtype="bf16", seed=5, k_offset_sigma=3.0)
    pr = _problem(w, smooth_q=True, qk_bits=4)
    q, k, v = generate(w)
    pre = oracle.prepass(pr, q, k, v, keep_fp32=True)
    _check_blocks(pre["kp"].astype(np.float64), pre["k8"], pre["k_scale"], 32, pr.Nkv)
    _check_blocks(pre["qp"].astype(np.float64), pre["q8"], pre["q_scale"], 1, pr.Nq)
    # V keeps its FP8 path: identical to the 8-bit run
    pre8 = oracle.prepass(_problem(w, smooth_q=True), q, k, v)
    assert np.array_equal(pre["v8"], pre8["v8"]) and np.array_equal(pre["v_scale"], pre8["v_scale"])


def _grid_inputs(B, H, N, D, blk, rng):
    """fp16 [B, H, N, D]: each block of `blk` tokens is 2^e times integers in
    [-7, 7] with a 7 in its first element."""
    ints = rng.integers(-7, 8, size=(B, H, N, D)).astype(np.float32)
    ints[:, :, ::blk, 0] = 7.0
    e = rng.integers(-4, 1, size=(B, H, (N + blk - 1) // blk)).astype(np.float32)
    a = np.repeat(2.0 ** e, blk, axis=2)[:, :, :N, None]
    return ints, (ints * a).astype(np.float32)


@pytest.mark.parametrize("causal", [False, True])
def test_int4_is_exact_on_the_4bit_grid(causal):
    B, Hq, Hkv, Nq, Nkv, D = 1, 4, 2, 200, 300 if not causal else 200, 64
    rng = np.random.default_rng(12)
    qi, Q = _grid_inputs(B, Hq, Nq, D, 1, rng)
    ki, K = _grid_inputs(B, Hkv, Nkv, D, 32, rng)
    V = rng.standard_normal((B, Hkv, Nkv, D)).astype(np.float32)
    q, k, v = _to_bits(Q, "fp16"), _to_bits(K, "fp16"), _to_bits(V, "fp16")
    w = random_problem(B, Hq, Hkv, Nq, Nkv, D, dtype="fp16")
    pr4 = _problem(w, is_causal=causal, smooth_k=False, qk_bits=4)
    pre4 = oracle.prepass(pr4, q, k, v, keep_fp32=True)
    assert np.array_equal(pre4["q8"], qi.astype(np.int8))
    assert np.array_equal(pre4["k8"], ki.astype(np.int8))
    tiles = oracle.all_tiles(pr4)
    out4 = oracle.attention_tiles(pr4, pre4, tiles)
    ref = oracle.attention_tiles(pr4, pre4, tiles, exact_mask=oracle.KEEP_QK)
    assert np.max(np.abs(out4 - ref)) <= 1e-12 * np.max(np.abs(ref))
    # the 8-bit codes of the same inputs are not exact (127/7 is no integer)
    pr8 = _problem(w, is_causal=causal, smooth_k=False)
    pre8 = oracle.prepass(pr8, q, k, v)
    assert not np.array_equal(pre8["q8"], (qi * 127 / 7).astype(np.int8))
    assert np.max(np.abs(oracle.attention_tiles(pr8, pre8, tiles) - ref)) > 0


@pytest.mark.parametrize("D", [64, 128])
def test_q_smoothing_keeps_the_int4_error_small(D):
    w = random_problem(1, 2, 2, 512, 1024, D, dtype="fp16", seed=3, k_offset_sigma=3.0)
    q, k, v = generate(w)
    off = np.random.default_rng(7).standard_normal((1, 2, 1, D)).astype(np.float32) * np.float32(3)
    q_off = _to_bits(q.view(np.float16).astype(np.float32) + off, "fp16")
    err = {}
    for name, qq in (("plain", q), ("offset", q_off)):
        for bits in (8, 4):
            for sq in (False, True):
                pr = _problem(w, qk_bits=bits, smooth_q=sq)
                tiles = oracle.all_tiles(pr)
                ex = oracle.exact_attention_tiles(pr, qq, k, v, tiles)
                err[name, bits, sq] = _rel_l1(oracle.attention_tiles(pr, oracle.prepass(pr, qq, k, v), tiles), ex)
    # 4 bits cost more than 8 on the same data
    for name in ("plain", "offset"):
        for sq in (False, True):
            assert err[name, 4, sq] > 3 * err[name, 8, sq]
    # a common channel offset in Q: smoothing Q at least halves the 4-bit error
    assert err["offset", 4, True] < 0.5 * err["offset", 4, False]
    # no offset: smoothing changes the 4-bit error by a few percent at most
    assert abs(err["plain", 4, True] - err["plain", 4, False]) < 0.05 * err["plain", 4, False]

"""Pins of the oracle's smoothing and quantisation steps.

Each check is computed independently of the oracle's C code (numpy on the
decoded inputs) and fails for the plausible mistakes: a mean over the wrong
axis, a wrong block size or block index, a scale that is not amax/127, the
wrong rounding rule, a ragged block that counts padding, a layout mix-up.
"""
import numpy as np
import pytest

import oracle
from quantized_attention_subtract_b200.workloads import generate, random_problem


def _problem(w, **kw):
    d = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, Nq=w.Nq, Nkv=w.Nkv, D=w.D, layout=w.layout, dtype=w.dtype,
             is_causal=w.is_causal, smooth_k=w.smooth_k, smooth_q=w.smooth_q, smooth_v=w.smooth_v)
    d.update(kw)
    return oracle.Problem(**d)


def _hnd(pr, x, H, N):
    x = oracle.to_double(pr, x)
    return x if pr.layout == "HND" else x.transpose(0, 2, 1, 3)


@pytest.fixture(scope="module")
def case():
    w = random_problem(2, 4, 2, 300, 200, 64, dtype="bf16", seed=5, k_offset_sigma=3.0)
    pr = _problem(w, smooth_q=True, smooth_v=True)
    q, k, v = generate(w)
    return pr, q, k, v, oracle.prepass(pr, q, k, v)


def test_mean_k_is_channel_mean_over_tokens(case):
    pr, q, k, v, pre = case
    K = _hnd(pr, k, pr.Hkv, pr.Nkv)
    want = K.mean(axis=2)  # over tokens, per (b, h, channel)
    # fixed point with 2^-24 resolution, then one fp32 rounding
    tol = 2.0 ** -25 + np.abs(want) * 2.0 ** -23
    assert np.all(np.abs(pre["mean_k"] - want) <= tol)


def test_smooth_k_off_gives_zero_mean(case):
    pr, q, k, v, _ = case
    pr0 = oracle.Problem(**{**pr.__dict__, "smooth_k": False})
    pre0 = oracle.prepass(pr0, q, k, v)
    assert np.all(pre0["mean_k"] == 0)
    K = _hnd(pr, k, pr.Hkv, pr.Nkv)
    assert np.array_equal(pre0["kp"].astype(np.float64), K)


def test_k_prime_is_k_minus_mean(case):
    pr, q, k, v, pre = case
    K = _hnd(pr, k, pr.Hkv, pr.Nkv)
    exact = K - pre["mean_k"][:, :, None, :].astype(np.float64)
    assert np.all(np.abs(pre["kp"] - exact) <= np.abs(exact) * 2.0 ** -24)


def _check_int8_blocks(x, codes, scales, blk, axis_len):
    """Blocks of `blk` tokens (all D channels) along axis -2, one scale each."""
    nb = (axis_len + blk - 1) // blk
    assert scales.shape[-1] == nb
    for i in range(nb):
        sl = slice(i * blk, min((i + 1) * blk, axis_len))
        xb, cb, s = x[..., sl, :], codes[..., sl, :].astype(np.float64), scales[..., i]
        if not np.any(s):
            continue
        amax = np.abs(xb).max(axis=(-2, -1))
        assert np.array_equal(s, (amax.astype(np.float32) / np.float32(127)))
        assert np.all(np.abs(cb) <= 127)
        assert np.all(np.abs(cb).max(axis=(-2, -1)) == 127)
        # round trip: |x - code*scale| <= scale/2 (plus fp32 slack on the reciprocal)
        err = np.abs(xb - cb * s[..., None, None])
        assert np.all(err <= s[..., None, None] * (0.5 + 2.0 ** -16))


def test_k_int8_blocks_of_32(case):
    pr, q, k, v, pre = case
    assert pre["k_scale"].shape[-1] == (pr.Nkv + 31) // 32
    _check_int8_blocks(pre["kp"].astype(np.float64), pre["k8"], pre["k_scale"], 32, pr.Nkv)


def test_q_int8_per_token_with_block_mean_smoothing(case):
    pr, q, k, v, pre = case
    Q = _hnd(pr, q, pr.Hq, pr.Nq)
    qp = np.empty_like(Q)
    for i in range(pr.nmb):
        sl = slice(i * 128, min((i + 1) * 128, pr.Nq))
        mean = Q[:, :, sl].mean(axis=2)
        assert np.all(np.abs(pre["mq"][:, :, i] - mean) <= 2.0 ** -25 + np.abs(mean) * 2.0 ** -23)
        qp[:, :, sl] = (Q[:, :, sl].astype(np.float32) - pre["mq"][:, :, i][:, :, None, :])
    assert pre["q_scale"].shape == (pr.B, pr.Hq, pr.Nq)
    _check_int8_blocks(qp, pre["q8"], pre["q_scale"], 1, pr.Nq)
    # the fp32 Q' the pre-pass hands to the error decomposition is the same
    pre32 = oracle.prepass(pr, q, k, v, keep_fp32=True)
    assert np.array_equal(pre32["qp"].astype(np.float64), qp)


def test_ragged_last_block_uses_only_valid_tokens():
    # The last K block has 8 tokens: its scale is the amax of those 8 only;
    # the last Q token's scale is its own amax.
    w = random_problem(1, 1, 1, 130, 72, 64, seed=9, k_offset_sigma=0.0)
    pr = _problem(w, smooth_k=False)
    q, k, v = generate(w)
    pre = oracle.prepass(pr, q, k, v)
    K = _hnd(pr, k, 1, 72)
    assert pre["k_scale"].shape[-1] == 3
    assert pre["k_scale"][0, 0, 2] == np.float32(np.abs(K[0, 0, 64:72]).max()) / np.float32(127)
    Q = _hnd(pr, q, 1, 130)
    assert pre["q_scale"][0, 0, 129] == np.float32(np.abs(Q[0, 0, 129]).max()) / np.float32(127)


def test_zero_block_has_zero_scale_and_codes():
    w = random_problem(1, 1, 1, 128, 128, 64, dtype="fp16", seed=1, k_offset_sigma=0.0)
    pr = _problem(w, smooth_k=False)
    q, k, v = generate(w)
    k = k.copy()
    k[0, 0, 64:96] = 0   # third K block all zero (fp16 +0 bits)
    q = q.copy()
    q[0, 0, 5] = 0       # query token 5 all zero
    v = v.copy()
    v[0, 0, :, 3] = 0    # channel 3 of V all zero
    pre = oracle.prepass(pr, q, k, v)
    assert pre["k_scale"][0, 0, 2] == 0 and np.all(pre["k8"][0, 0, 64:96] == 0)
    assert pre["k_scale"][0, 0, 1] > 0 and pre["k_scale"][0, 0, 3] > 0
    assert pre["q_scale"][0, 0, 5] == 0 and np.all(pre["q8"][0, 0, 5] == 0)
    assert pre["v_scale"][0, 0, 3] == 0 and np.all(pre["v8"][0, 0, :, 3] == 0)


def test_v_fp8_per_channel(case):
    pr, q, k, v, pre = case
    V = _hnd(pr, v, pr.Hkv, pr.Nkv)
    mv = V.mean(axis=2)
    assert np.all(np.abs(pre["mean_v"] - mv) <= 2.0 ** -25 + np.abs(mv) * 2.0 ** -23)
    vp = V.astype(np.float32) - pre["mean_v"][:, :, None, :]
    amax = np.abs(vp).max(axis=2)
    assert np.array_equal(pre["v_scale"], amax.astype(np.float32) / np.float32(448))
    table = oracle.e4m3_decode_table()
    dec = table[pre["v8"]] * pre["v_scale"][:, :, None, :]
    s = pre["v_scale"][:, :, None, :].astype(np.float64)
    # e4m3 round-to-nearest: relative 2^-4 in the normal range, 2^-10 * 448 * scale... in units of
    # the channel scale the subnormal step is 2^-9, so the absolute error there is <= 2^-10 * scale
    err = np.abs(dec - vp)
    assert np.all(err <= np.abs(vp) * 2.0 ** -4 * (1 + 2.0 ** -20) + 2.0 ** -10 * s)
    # every nonzero channel uses the top code 448 somewhere
    codes = pre["v8"] & 0x7F
    assert np.all(codes.max(axis=2) == 0x7E)


def test_prepass_is_layout_invariant():
    w = random_problem(2, 4, 2, 257, 190, 96, dtype="fp16", seed=11)
    pr_h = _problem(w, smooth_q=True, smooth_v=True)
    qh, kh, vh = generate(w)
    qn, kn, vn = generate(w.with_(layout="NHD"))
    pr_n = _problem(w.with_(layout="NHD"), smooth_q=True, smooth_v=True)
    a, b = oracle.prepass(pr_h, qh, kh, vh), oracle.prepass(pr_n, qn, kn, vn)
    for key in a:
        assert np.array_equal(a[key], b[key]), key

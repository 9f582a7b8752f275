"""Pins of the oracle's attention: invariants, identities, special cases, bounds.

- smooth_k invariant: subtracting the per-channel K mean shifts every logit of
  a row by the same constant, so fp64 softmax attention is unchanged
  ("sageattention" package page, Quickstart: smooth_k=True by default).
- Q smoothing: Q'K'^T + 1 dS^T restores Q K'^T exactly ("SageAttention2:
  Technical report", section 2: subtract the channel mean of Q and V).
- V smoothing: P(V - 1 mu^T) + 1 mu^T = P V for row-stochastic P (same section).
- Special cases with a closed form: Q = 0 gives the mean of the (dequantised)
  visible V rows (prefix means when causal); Nkv = 1 gives that row; constant
  V gives the constant up to the FP8 rounding of P.
- The fp64 exact attention equals PyTorch's scaled_dot_product_attention in
  fp64 (library routine), including causal masking and GQA.
- With every quantisation step switched off (P, V and Q K^T unquantised) the
  tiled online softmax is exact softmax attention: a dropped rescale, a wrong
  running max, a masking or GQA index error would all show here.
- Error decomposition on iid inputs: FP8 rounding of P alone and of V alone
  each cost the closed-form rms relative error of e4m3 round-to-nearest
  (2^-3/sqrt(12) * sqrt(3/(8 ln 2)) = 0.0265 for log-uniform mantissas), the
  two together their quadrature sum, and INT8 Q K^T (per-token Q, 32-key K
  scales) well below either.
- The running max is the plain one: each tile's largest logit gets the FP8
  code of 448 exactly and earlier tiles are rescaled by 2^(m_old - m_new).
- The quantised mirror stays within the error the FP8/INT8 steps allow of the
  exact result (relative L1 <= 0.06, cosine >= 0.998 on iid data), also when
  block scales differ by orders of magnitude and when the running max grows
  tile after tile.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_attention_subtract_b200.workloads import generate, random_problem


def _problem(w, **kw):
    d = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, Nq=w.Nq, Nkv=w.Nkv, D=w.D, layout=w.layout, dtype=w.dtype,
             is_causal=w.is_causal, smooth_k=w.smooth_k, smooth_q=w.smooth_q, smooth_v=w.smooth_v)
    d.update(kw)
    return oracle.Problem(**d)


def _hnd(pr, x):
    x = oracle.to_double(pr, x)
    return x if pr.layout == "HND" else x.transpose(0, 2, 1, 3)


def _tiled(pr, full_hnd):
    """[B,H,N,D] -> [n_tiles,128,D] in all_tiles order."""
    t = oracle.all_tiles(pr)
    out = np.zeros((len(t), 128, pr.D))
    for n, (b, h, qt) in enumerate(t):
        i0, i1 = qt * 128, min(qt * 128 + 128, pr.Nq)
        out[n, : i1 - i0] = full_hnd[b, h, i0:i1]
    return out


def _softmax_attn(Q, K, V, scale, causal, group):
    K = np.repeat(K, group, axis=1)
    V = np.repeat(V, group, axis=1)
    s = np.einsum("bhid,bhjd->bhij", Q, K) * scale
    if causal:
        i = np.arange(Q.shape[2])[:, None]
        j = np.arange(K.shape[2])[None, :]
        s = np.where(j <= i, s, -np.inf)
    s = s - s.max(-1, keepdims=True)
    p = np.exp(s)
    return np.einsum("bhij,bhjd->bhid", p / p.sum(-1, keepdims=True), V)


def _rel_l1(a, b):
    return np.abs(a - b).sum() / np.abs(b).sum()


def _cos(a, b):
    return (a * b).sum() / np.linalg.norm(a) / np.linalg.norm(b)


@pytest.mark.parametrize("causal", [False, True])
def test_exact_attention_matches_torch_sdpa_fp64(causal):
    w = random_problem(2, 4, 2, 200, 200 if causal else 333, 64, dtype="fp16", seed=4)
    pr = _problem(w, is_causal=causal)
    q, k, v = generate(w)
    Q, K, V = (torch.from_numpy(_hnd(pr, x)) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q, K, V, is_causal=causal, scale=float(pr.resolved_sm_scale()), enable_gqa=True).numpy()
    got = oracle.exact_attention_tiles(pr, q, k, v, oracle.all_tiles(pr))
    assert np.max(np.abs(got - _tiled(pr, ref))) < 1e-12


def test_smooth_k_invariant_fp64():
    w = random_problem(1, 2, 2, 256, 256, 64, dtype="fp16", seed=0, k_offset_sigma=3.0)
    pr = _problem(w)
    q, k, v = generate(w)
    pre = oracle.prepass(pr, q, k, v)
    Q, K, V = _hnd(pr, q), _hnd(pr, k), _hnd(pr, v)
    s = float(pr.resolved_sm_scale())
    a = _softmax_attn(Q, K, V, s, False, 1)
    b = _softmax_attn(Q, K - pre["mean_k"][:, :, None, :], V, s, False, 1)
    assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(a))
    # subtracting a per-*token* quantity instead would not be invariant
    c = _softmax_attn(Q, K - K.mean(axis=3, keepdims=True), V, s, False, 1)
    assert np.max(np.abs(a - c)) > 1e-3


def test_q_smoothing_correction_restores_qk():
    w = random_problem(1, 4, 2, 300, 200, 96, dtype="bf16", seed=6, k_offset_sigma=3.0)
    pr = _problem(w, smooth_q=True)
    q, k, v = generate(w)
    pre = oracle.prepass(pr, q, k, v)
    Q = _hnd(pr, q)
    for b, h, qt in [(0, 0, 0), (0, 3, 2), (0, 1, 1)]:
        kp = pre["kp"][0, h // 2].astype(np.float64)
        i0, i1 = qt * 128, min(qt * 128 + 128, pr.Nq)
        Qb = Q[b, h, i0:i1]
        mq = pre["mq"][b, h, qt].astype(np.float64)
        dS = oracle.delta_s(pr, pre, b, h, qt)
        lhs = (Qb - mq) @ kp.T + dS[None, :]
        rhs = Qb @ kp.T
        assert np.max(np.abs(lhs - rhs)) <= 1e-12 * np.max(np.abs(rhs))
        # dropping the correction is far off
        assert np.max(np.abs((Qb - mq) @ kp.T - rhs)) > 1e-3


def test_v_smoothing_identity():
    w = random_problem(1, 2, 2, 128, 200, 64, dtype="fp16", seed=7)
    pr = _problem(w, smooth_v=True)
    q, k, v = generate(w)
    pre = oracle.prepass(pr, q, k, v)
    V = _hnd(pr, v)[0, 0]
    mu = pre["mean_v"][0, 0].astype(np.float64)
    rng = np.random.default_rng(0)
    P = rng.random((128, 200))
    P /= P.sum(1, keepdims=True)
    assert np.max(np.abs(P @ (V - mu) + mu - P @ V)) < 1e-12


@pytest.mark.parametrize("causal,layout,Nq,Nkv,Hq,Hkv,D", [
    (False, "HND", 256, 200, 4, 2, 64),
    (True, "HND", 300, 300, 4, 1, 128),
    (True, "NHD", 260, 260, 2, 2, 96),
    (False, "NHD", 130, 700, 6, 3, 64),
])
def test_zero_q_gives_mean_of_visible_v(causal, layout, Nq, Nkv, Hq, Hkv, D):
    w = random_problem(2, Hq, Hkv, Nq, Nkv, D, layout=layout, dtype="bf16", seed=8)
    pr = _problem(w, is_causal=causal, smooth_v=True)
    q, k, v = generate(w)
    q = np.zeros_like(q)
    pre = oracle.prepass(pr, q, k, v)
    table = oracle.e4m3_decode_table()
    Vd = table[pre["v8"]] * pre["v_scale"][:, :, None, :] + pre["mean_v"][:, :, None, :]
    Vd = np.repeat(Vd, Hq // Hkv, axis=1)
    if causal:
        want = np.cumsum(Vd, axis=2)[:, :, :Nq] / np.arange(1, Nq + 1)[None, None, :, None]
    else:
        want = np.broadcast_to(Vd.mean(axis=2, keepdims=True), (2, Hq, Nq, D))
    got = oracle.attention_tiles(pr, pre, oracle.all_tiles(pr))
    assert np.max(np.abs(got - _tiled(pr, want))) <= 1e-6 * np.max(np.abs(want))


def test_single_key_gives_that_row():
    w = random_problem(1, 2, 1, 200, 1, 128, dtype="fp16", seed=9)
    pr = _problem(w)
    q, k, v = generate(w)
    pre = oracle.prepass(pr, q, k, v)
    table = oracle.e4m3_decode_table()
    row = table[pre["v8"][0, 0, 0]] * pre["v_scale"][0, 0]
    got = oracle.attention_tiles(pr, pre, oracle.all_tiles(pr))
    valid = np.concatenate([got[0], got[1, :72], got[2], got[3, :72]])
    assert np.max(np.abs(valid - row)) <= 1e-6 * np.max(np.abs(row))


def test_constant_v_gives_the_constant():
    w = random_problem(1, 2, 2, 256, 500, 64, dtype="fp16", seed=10)
    pr = _problem(w)
    q, k, v = generate(w)
    const = np.linspace(-3, 3, 64).astype(np.float16)
    v = np.broadcast_to(const.view(np.uint16), v.shape).copy()
    pre = oracle.prepass(pr, q, k, v)
    got = oracle.attention_tiles(pr, pre, oracle.all_tiles(pr))
    c = const.astype(np.float64)
    # sum of FP8-rounded p over sum of p is within the e4m3 relative step 2^-4 of 1
    assert np.all(np.abs(got - c) <= 2.0 ** -4 * np.abs(c) + 1e-12)


CASES = [
    dict(args=(1, 2, 2, 256, 256, 64), dtype="fp16"),
    dict(args=(2, 4, 2, 300, 200, 96), dtype="bf16"),
    dict(args=(1, 4, 1, 384, 384, 128), dtype="bf16", is_causal=True),
    dict(args=(1, 2, 2, 256, 512, 64), dtype="fp16", smooth_k=False),
    dict(args=(1, 2, 2, 256, 512, 64), dtype="fp16", smooth_q=True, smooth_v=True),
    dict(args=(1, 2, 2, 200, 390, 64), dtype="bf16", layout="NHD", is_causal=True),
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_mirror_within_quantisation_error_of_exact(case):
    flags = {k: v for k, v in case.items() if k in ("is_causal", "smooth_k", "smooth_q", "smooth_v")}
    w = random_problem(*case["args"], layout=case.get("layout", "HND"), dtype=case["dtype"], seed=3,
                       k_offset_sigma=3.0)
    pr = _problem(w, **flags)
    q, k, v = generate(w)
    pre = oracle.prepass(pr, q, k, v)
    t = oracle.all_tiles(pr)
    m = oracle.attention_tiles(pr, pre, t)
    e = oracle.exact_attention_tiles(pr, q, k, v, t)
    assert _rel_l1(m, e) <= 0.06 and _cos(m, e) >= 0.998


def test_mirror_uses_the_right_block_scales():
    # K blocks (32 tokens) and Q tokens with magnitudes that differ by orders
    # of magnitude: a wrong block or token index in the scale lookup changes
    # logits by large factors.
    w = random_problem(1, 2, 2, 384, 384, 64, dtype="fp16", seed=12, k_offset_sigma=0.0)
    pr = _problem(w, smooth_k=False)
    q, k, v = generate(w)
    Q, K = oracle.to_double(pr, q), oracle.to_double(pr, k)
    rng = np.random.default_rng(3)
    kscale = 10.0 ** rng.uniform(-1.5, 0.5, 384 // 32)
    qscale = 10.0 ** rng.uniform(-1.0, 0.3, 384)
    K = K * np.repeat(kscale, 32)[None, None, :, None]
    Q = Q * qscale[None, None, :, None]
    q = Q.astype(np.float16).view(np.uint16)
    k = K.astype(np.float16).view(np.uint16)
    pre = oracle.prepass(pr, q, k, v)
    t = oracle.all_tiles(pr)
    m = oracle.attention_tiles(pr, pre, t)
    e = oracle.exact_attention_tiles(pr, q, k, v, t)
    assert _rel_l1(m, e) <= 0.06 and _cos(m, e) >= 0.998


def test_mirror_rescales_when_max_grows():
    # Logits rise tile after tile, so the running max grows in every KV tile
    # and the O / l rescaling is exercised on every step.
    w = random_problem(1, 1, 1, 128, 1024, 64, dtype="fp16", seed=13, k_offset_sigma=0.0)
    pr = _problem(w, smooth_k=False)
    q, k, v = generate(w)
    rng = np.random.default_rng(1)
    u = rng.standard_normal(64)
    u /= np.linalg.norm(u)
    Q = 0.3 * rng.standard_normal((1, 1, 128, 64)) + 2.0 * u
    ramp = np.linspace(0, 6.0, 1024)[:, None]
    K = 0.3 * rng.standard_normal((1, 1, 1024, 64)) + ramp * u
    q = Q.astype(np.float16).view(np.uint16)
    k = K.astype(np.float16).view(np.uint16)
    pre = oracle.prepass(pr, q, k, v)
    t = oracle.all_tiles(pr)
    m = oracle.attention_tiles(pr, pre, t)
    e = oracle.exact_attention_tiles(pr, q, k, v, t)
    assert _rel_l1(m, e) <= 0.06 and _cos(m, e) >= 0.998


def test_mirror_is_layout_invariant():
    w = random_problem(2, 4, 2, 200, 300, 64, dtype="bf16", seed=14)
    pr_h, pr_n = _problem(w, is_causal=False), _problem(w.with_(layout="NHD"))
    a = oracle.attention_tiles(pr_h, oracle.prepass(pr_h, *generate(w)), oracle.all_tiles(pr_h))
    b = oracle.attention_tiles(pr_n, oracle.prepass(pr_n, *generate(w.with_(layout="NHD"))),
                               oracle.all_tiles(pr_n))
    assert np.array_equal(a, b)


def test_uncertainty_is_zero_when_p_codes_are_exact_and_small_otherwise():
    # Q = 0: every P equals 448 exactly, so no code is ambiguous.
    w = random_problem(1, 2, 2, 256, 300, 64, dtype="fp16", seed=15)
    pr = _problem(w)
    q, k, v = generate(w)
    pre = oracle.prepass(pr, np.zeros_like(q), k, v)
    _, unc = oracle.attention_tiles(pr, pre, oracle.all_tiles(pr), with_uncertainty=True)
    assert np.all(unc == 0)
    # random inputs: a few ambiguous codes (a fraction of the outputs sees
    # one of its 300 keys ambiguous), each worth at most one e4m3 step
    pre = oracle.prepass(pr, q, k, v)
    out, unc = oracle.attention_tiles(pr, pre, oracle.all_tiles(pr), with_uncertainty=True)
    assert np.all(unc >= 0)
    assert 0 < (unc > 0).mean() < 0.25
    assert unc.max() < 0.01 * np.abs(out).max()
    assert unc.mean() < 1e-3 * np.abs(out).mean()
    # the mirror itself is unchanged by asking for the bound
    assert np.array_equal(out, oracle.attention_tiles(pr, pre, oracle.all_tiles(pr)))


ALL_EXACT = oracle.KEEP_P | oracle.KEEP_V | oracle.KEEP_QK

EXACT_CASES = [
    dict(args=(1, 2, 2, 256, 256, 64), dtype="fp16"),
    dict(args=(2, 4, 2, 300, 520, 96), dtype="bf16", layout="NHD"),
    dict(args=(1, 4, 1, 384, 384, 128), dtype="bf16", is_causal=True),
    dict(args=(1, 2, 2, 200, 700, 64), dtype="fp16", is_causal=True),
    dict(args=(1, 2, 2, 256, 512, 128), dtype="fp16", smooth_q=True, smooth_v=True),
    dict(args=(1, 2, 1, 129, 300, 64), dtype="bf16", smooth_k=False, smooth_v=True),
]


@pytest.mark.parametrize("case", EXACT_CASES, ids=[str(i) for i in range(len(EXACT_CASES))])
def test_mirror_with_nothing_quantised_is_exact_attention(case):
    flags = {k: v for k, v in case.items() if k in ("is_causal", "smooth_k", "smooth_q", "smooth_v")}
    w = random_problem(*case["args"], layout=case.get("layout", "HND"), dtype=case["dtype"], seed=17,
                       k_offset_sigma=3.0)
    pr = _problem(w, **flags)
    q, k, v = generate(w)
    pre = oracle.prepass(pr, q, k, v, keep_fp32=True)
    t = oracle.all_tiles(pr)
    m = oracle.attention_tiles(pr, pre, t, exact_mask=ALL_EXACT)
    e = oracle.exact_attention_tiles(pr, q, k, v, t)
    rows = np.zeros((len(t), 128), bool)
    for n, (_, _, qt) in enumerate(t):
        rows[n, : max(0, min(128, pr.Nq - 128 * qt))] = True
    # only the fp32 rounding of the smoothed inputs (Q - mq, K - mean_k,
    # V - mean_v) separates the two
    assert np.max(np.abs(m[rows] - e[rows])) <= 1e-5 * np.max(np.abs(e[rows]))
    # quantising anything moves it by far more than that
    assert np.max(np.abs(oracle.attention_tiles(pr, pre, t)[rows] - e[rows])) > 1e-3


# rms relative error of e4m3 round-to-nearest for log-uniform mantissas:
# step 2^-3 relative to the binade start, error uniform in half a step,
# E[2^-2u] = 3 / (8 ln 2) over u ~ U(0, 1)
E4M3_RMS = 2.0 ** -3 / np.sqrt(12.0) * np.sqrt(3.0 / (8.0 * np.log(2.0)))


def test_error_decomposition_iid():
    w = random_problem(1, 2, 2, 768, 1024, 128, dtype="bf16", seed=18, k_offset_sigma=3.0)
    pr = _problem(w)
    q, k, v = generate(w)
    pre = oracle.prepass(pr, q, k, v, keep_fp32=True)
    t = oracle.all_tiles(pr)
    e = oracle.exact_attention_tiles(pr, q, k, v, t)
    err = {}
    for name, keep in dict(p=ALL_EXACT ^ oracle.KEEP_P, v=ALL_EXACT ^ oracle.KEEP_V,
                           qk=ALL_EXACT ^ oracle.KEEP_QK, pv=oracle.KEEP_QK, all=0).items():
        err[name] = _rel_l1(oracle.attention_tiles(pr, pre, t, exact_mask=keep), e)
    # FP8 P and FP8 V alone: the e4m3 rms error (P a little less: each row's
    # maximum gets the exact code 448)
    assert 0.80 * E4M3_RMS <= err["p"] <= 1.05 * E4M3_RMS, err
    assert 0.90 * E4M3_RMS <= err["v"] <= 1.10 * E4M3_RMS, err
    # independent roundings add in quadrature
    assert abs(err["pv"] - np.hypot(err["p"], err["v"])) <= 0.08 * err["pv"], err
    # INT8 Q K^T with per-token Q and 32-key K scales is the small part
    assert err["qk"] <= 0.5 * err["p"], err
    total = np.sqrt(err["p"] ** 2 + err["v"] ** 2 + err["qk"] ** 2)
    assert abs(err["all"] - total) <= 0.10 * total, err
    assert err["all"] <= 0.045, err


def test_running_max_is_the_plain_one():
    # One query row, two KV tiles.  The largest logit of tile 1 sits at key
    # j1, that of tile 2 at key j2 with s(j2) - s(j1) = d in (0, 1).  V is an
    # indicator: channel 0 of key j2, channel 1 of key j1 (both decode to
    # exactly 1).  With the plain running max each tile's largest logit gets
    # P code 448 and tile 1's contribution is rescaled by 2^-d when tile 2
    # raises the max, so o_1 / o_0 = 2^(s(j1) - s(j2)) exactly; a max raised
    # only past a threshold would leave tile 1 unscaled and give key j2 a code
    # other than 448.
    D, Nkv = 64, 256
    w = random_problem(1, 1, 1, 1, Nkv, D, dtype="fp16", seed=19, k_offset_sigma=0.0)
    pr = _problem(w, smooth_k=False)
    qv = np.zeros((1, 1, 1, D))
    qv[0, 0, 0, 0] = 1.0
    kv = np.zeros((1, 1, Nkv, D))
    kv[0, 0, :, 0] = np.linspace(-2.0, 1.0, Nkv)       # logits rise with j
    j1, j2 = 100, 200
    kv[0, 0, j1, 0] = 2.0                                # tile 1's maximum
    kv[0, 0, j2, 0] = 2.5                                # tile 2's, higher by less than 1 in log2
    kv[0, 0, :, 1] = 1.0                                 # keep every K block's amax equal
    vv = np.zeros((1, 1, Nkv, D))
    vv[0, 0, j2, 0] = 1.0
    vv[0, 0, j1, 1] = 1.0
    q, k, v = (x.astype(np.float16).view(np.uint16) for x in (qv, kv, vv))
    pre = oracle.prepass(pr, q, k, v)
    o = oracle.attention_tiles(pr, pre, oracle.all_tiles(pr))[0, 0]
    S = pre["k8"][0, 0].astype(np.int64) @ pre["q8"][0, 0, 0].astype(np.int64)
    c = (pre["q_scale"][0, 0, 0].astype(np.float64) * pre["k_scale"][0, 0].astype(np.float64)
         * float(pr.resolved_sm_scale()) / np.log(2.0))
    s = S * np.repeat(c, 32)
    assert np.argmax(s[:128]) == j1 and np.argmax(s) == j2 and 0 < s[j2] - s[j1] < 1
    assert abs(o[1] / o[0] - 2.0 ** (s[j1] - s[j2])) <= 1e-12

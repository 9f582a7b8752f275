"""Pins of the oracle's number formats against their definitions and library routines.

The oracle's e4m3 encoder decides every FP8 code of V and P; a wrong rounding
direction, tie rule, subnormal grid or saturation point would shift the whole
reference.  These checks tie it to (a) the format's printed reference points,
(b) brute-force nearest-value search over the decoded code table, and (c)
PyTorch's own float8_e4m3fn conversion inside the finite range.
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_points.txt")


def _golden():
    pts = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        c, v = line.split()
        pts.append((int(c, 16), float(v)))
    return pts


def test_e4m3_decode_matches_format_points():
    table = oracle.e4m3_decode_table()
    for code, value in _golden():
        assert table[code] == value, (hex(code), table[code], value)
        assert np.signbit(table[code]) == np.signbit(value)
    assert np.isnan(table[0x7F]) and np.isnan(table[0xFF])
    assert np.isnan(table).sum() == 2


def test_e4m3_decode_is_monotone_and_symmetric():
    table = oracle.e4m3_decode_table()
    pos = table[0x00:0x7F]
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(table[0x80:0xFF], -pos)


def _nearest_even(x, table):
    """Brute force: nearest finite code; ties to the code with even mantissa; |x| > 448 -> +-448."""
    finite = [c for c in range(256) if not np.isnan(table[c])]
    out = np.empty(len(x), np.uint8)
    for n, xv in enumerate(x):
        if abs(xv) >= 448:
            out[n] = 0x7E if xv > 0 else 0xFE
            continue
        same_sign = [c for c in finite if (c >> 7) == (1 if np.signbit(xv) else 0)]
        d = np.array([abs(table[c] - xv) for c in same_sign])
        best = d.min()
        cands = [same_sign[i] for i in np.nonzero(d == best)[0]]
        if len(cands) > 1:
            cands = [c for c in cands if (c & 1) == 0]
        out[n] = cands[0]
    return out


def test_e4m3_encode_equals_bruteforce_nearest():
    table = oracle.e4m3_decode_table()
    pos = table[0x00:0x7F]
    mids = (pos[1:] + pos[:-1]) / 2
    rng = np.random.default_rng(1)
    x = np.concatenate([
        pos, mids, np.nextafter(mids, 0), np.nextafter(mids, 1000),
        2.0 ** rng.uniform(-12, 9.5, 3000), [448.0, 449.0, 463.9, 464.0, 465.0, 1e6, 0.0],
        rng.uniform(0, 2 ** -9, 200),
    ])
    x = np.concatenate([x, -x])
    got = oracle.e4m3_encode(x)
    want = _nearest_even(x, table)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(x[i], got[i], want[i]) for i in bad[:10]]


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(2)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 50,
        (2.0 ** rng.uniform(-16, 8.8, 200000)).astype(np.float32),
        np.arange(-463, 464, 0.125, dtype=np.float32),
    ])
    x = x[np.abs(x) < 464]  # torch does not saturate; above 464 it gives NaN
    got = oracle.e4m3_encode_f32(x)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, want)


def test_e4m3_saturates_finite():
    got = oracle.e4m3_encode(np.array([448.0, 500.0, 1e30, -1e30, -470.0]))
    assert list(got) == [0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_16bit_decoders_match_library(dtype):
    pr = oracle.Problem(1, 1, 1, 1, 1, 64, dtype=dtype)
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.to_double(pr, bits)
    if dtype == "fp16":
        want = bits.view(np.float16).astype(np.float64)
    else:
        want = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).double().numpy()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])


def test_output_rounding_matches_library():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(100000) * 10, 2.0 ** rng.uniform(-30, 15, 20000),
                        [65504.0, 65519.9, 65520.0, 1e-8, 3e-8, 0.0, -0.0]])
    pr16 = oracle.Problem(1, 1, 1, 1, 1, 64, dtype="fp16")
    assert np.array_equal(oracle.round_output(pr16, x), x.astype(np.float16).view(np.uint16))
    # bf16: compare on float32-representable inputs, where torch's float->bf16 is a single rounding
    xf = x.astype(np.float32)
    xf = xf[np.isfinite(xf)]
    prb = oracle.Problem(1, 1, 1, 1, 1, 64, dtype="bf16")
    want = torch.from_numpy(xf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.round_output(prb, xf.astype(np.float64)), want)

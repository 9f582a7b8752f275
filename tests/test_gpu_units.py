"""GPU unit checks of the kernel building blocks, through the C ABI.

- FP8 e4m3 conversion: the kernel's conversion (used for V and P) equals the
  oracle's encoder written from the format definition, including byte order.
- A bounded wait that nothing completes reports SAGE_ERR_DEVICE_TIMEOUT and
  leaves the context usable.
- S tiles from the INT8 tensor-core path equal int64 dot products of the codes.
- A P V tile from the FP8 tensor-core path equals the fp64 product of the
  decoded codes up to fp32 accumulation rounding (no lossy accumulator).
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_attention_subtract_b200 import binding
from quantized_attention_subtract_b200.workloads import generate, random_problem

from _common import DeviceRun, oracle_problem

pytestmark = pytest.mark.gpu


def test_e4m3_conversion_matches_oracle_sample():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(1 << 20).astype(np.float32) * 100,
        (2.0 ** rng.uniform(-20, 10, 1 << 20)).astype(np.float32),
        np.array([0.0, -0.0, 448.0, 464.0, 1e30, -1e30, np.inf, -np.inf, 2 ** -9, 2 ** -10,
                  3 * 2 ** -11, 0.0146484375], np.float32),
    ])
    x = np.concatenate([x, -x])
    got = binding.debug_e4m3(torch.from_numpy(x).cuda()).cpu().numpy()
    assert np.array_equal(got, oracle.e4m3_encode_f32(x))


def test_e4m3_conversion_exhaustive():
    """Every fp32 bit pattern except NaNs, in chunks of 2^26."""
    chunk = 1 << 26
    base = np.arange(chunk, dtype=np.uint32)
    for c in range((1 << 32) // chunk):
        x = (base + np.uint32(c * chunk)).view(np.float32)
        keep = ~np.isnan(x)
        x = x[keep]
        got = binding.debug_e4m3(torch.from_numpy(x).cuda()).cpu().numpy()
        want = oracle.e4m3_encode_f32(x)
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, (c, [(float(x[i]), int(got[i]), int(want[i])) for i in bad[:5]])


def test_bounded_wait_reports_timeout_and_context_survives():
    st = torch.zeros(4, dtype=torch.int32, device="cuda")
    binding.debug_wait_timeout(st)
    torch.cuda.synchronize()
    assert int(st[0]) == 5  # SAGE_ERR_DEVICE_TIMEOUT
    w = random_problem(1, 2, 2, 128, 128, 64, seed=1)
    g = DeviceRun(w, *generate(w))
    assert torch.isfinite(g.out.float()).all()


@pytest.mark.parametrize("D,Nq,Nkv,layout", [(64, 256, 300, "HND"), (96, 130, 257, "NHD"),
                                             (128, 384, 200, "HND")])
def test_s_tiles_bit_exact(D, Nq, Nkv, layout):
    w = random_problem(2, 4, 2, Nq, Nkv, D, layout=layout, dtype="bf16", seed=D)
    q, k, v = generate(w)
    pre = oracle.prepass(oracle_problem(w), q, k, v)
    g = DeviceRun(w, q, k, v, run_attention=False)
    nqt, nkt = (Nq + 127) // 128, (Nkv + 127) // 128
    for b, h, qt, kt in [(0, 0, 0, 0), (1, 3, nqt - 1, nkt - 1), (0, 2, nqt - 1, 0), (1, 1, 0, nkt - 1)]:
        s = binding.debug_dump_s(g.p, b, h, qt, kt, "cuda").cpu().numpy().astype(np.int64)
        qb = np.zeros((128, D), np.int64)
        kb = np.zeros((128, D), np.int64)
        rq = pre["q8"][b, h, qt * 128: qt * 128 + 128]
        rk = pre["k8"][b, h // 2, kt * 128: kt * 128 + 128]
        qb[: len(rq)] = rq
        kb[: len(rk)] = rk
        assert np.array_equal(s, qb @ kb.T), (b, h, qt, kt)


@pytest.mark.parametrize("D", [64, 96, 128])
def test_pv_tile_fp32_accumulation(D):
    w = random_problem(1, 1, 1, 128, 256, D, dtype="fp16", seed=3)
    q, k, v = generate(w)
    pre = oracle.prepass(oracle_problem(w), q, k, v)
    g = DeviceRun(w, q, k, v, run_attention=False)
    rng = np.random.default_rng(D)
    table = oracle.e4m3_decode_table()
    # random non-negative finite codes, as P is
    p8 = rng.integers(0, 0x7F, size=(128, 128)).astype(np.uint8)
    for kt in range(2):
        o = binding.debug_pv(g.p, 0, 0, kt, torch.from_numpy(p8).cuda(), "cuda").cpu().numpy()
        vt = table[pre["v8"][0, 0, kt * 128: kt * 128 + 128]]
        want = table[p8] @ vt
        scale = (np.abs(table[p8]) @ np.abs(vt)) + 1e-30
        # within the worst case of 128 sequential fp32 additions; a reduced-
        # precision accumulator (about 14 mantissa bits) would be ~10x above
        assert np.max(np.abs(o - want) / scale) <= 128 * 2.0 ** -24, kt


def test_mma_loop_runs():
    sink = torch.zeros(149, dtype=torch.int32, device="cuda")
    binding.debug_mma_loop(148, 64, sink)
    torch.cuda.synchronize()
    assert int(sink[148]) == 0

"""GPU unit checks of the kernel building blocks, through the C ABI.

- FP8 e4m3 conversion: the kernel's conversion (used for V and P) equals the
  oracle's encoder written from the format definition, including byte order.
- A bounded wait that nothing completes reports SAGE_ERR_DEVICE_TIMEOUT and
  leaves the context usable.
- The int32 S tiles the production attention kernel's softmax warps read
  from tensor memory equal int64 dot products of the INT8 codes.
- The kernel's exp2 (ex2.approx.ftz.f32) stays within the relative error the
  oracle allows a hardware exp2 (2^-21) over the arguments the softmax uses.
- The 8-bit MMA loop (INT8 and FP8 kinds) runs and reports no failure.
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


@pytest.mark.parametrize("D,Nq,Nkv,layout,causal", [(64, 256, 300, "HND", False),
                                                    (96, 130, 257, "NHD", False),
                                                    (128, 384, 200, "HND", False),
                                                    (128, 520, 520, "HND", True)])
def test_s_tiles_bit_exact(D, Nq, Nkv, layout, causal):
    """S tiles as the attention kernel's softmax warps read them from tensor
    memory (an S-dump build of the same kernel), against int64 dot products
    of the INT8 codes, bit for bit; tiles of both query tiles of a pair,
    ragged key tiles and (causal) diagonal tiles."""
    w = random_problem(2, 4, 2, Nq, Nkv, D, layout=layout, dtype="bf16", seed=D,
                       is_causal=causal)
    q, k, v = generate(w)
    pre = oracle.prepass(oracle_problem(w), q, k, v)
    g = DeviceRun(w, q, k, v, run_attention=False)
    nqt, nkt = (Nq + 127) // 128, (Nkv + 127) // 128
    cases = [(0, 0, 0, 0), (1, 3, nqt - 1, nkt - 1), (0, 2, nqt - 1, 0), (1, 1, 0, nkt - 1),
             (0, 1, 1, nkt - 1)]
    for b, h, qt, kt in cases:
        s = binding.debug_dump_s(g.p, b, h, qt, kt, "cuda").cpu().numpy().astype(np.int64)
        torch.cuda.synchronize()
        assert binding.device_status(g.p) == 0
        if causal and kt * 128 > min(qt * 128 + 127, Nq - 1):
            assert np.all(s == -1), (b, h, qt, kt)   # a skipped tile is not computed
            continue
        qb = np.zeros((128, D), np.int64)
        kb = np.zeros((128, D), np.int64)
        rq = pre["q8"][b, h, qt * 128: qt * 128 + 128]
        rk = pre["k8"][b, h // 2, kt * 128: kt * 128 + 128]
        qb[: len(rq)] = rq
        kb[: len(rk)] = rk
        assert np.array_equal(s, qb @ kb.T), (b, h, qt, kt)


def test_ex2_error_within_the_oracle_allowance():
    """The relative error of the kernel's exp2 against fp64 exp2 over the
    arguments whose result can reach an FP8 code of P other than 0
    (t = s - m + log2(448) in [-20, 8.81]: e4m3's smallest subnormal is
    2^-9), at most the 2^-21 the oracle allows a hardware exp2 when it marks
    ambiguous FP8 codes of P."""
    rng = np.random.default_rng(0)
    t = np.concatenate([
        np.linspace(-20.0, 9.0, 1 << 22, dtype=np.float32),
        rng.uniform(-20.0, 9.0, 1 << 22).astype(np.float32),
        # every fp32 value in [8, 9): the top binade, where rounding the
        # argument matters most
        (np.arange(1 << 20, dtype=np.uint32) * np.uint32(8) + np.float32(8.0).view(np.uint32)).view(np.float32),
    ])
    got = binding.debug_ex2(torch.from_numpy(t).cuda()).cpu().numpy().astype(np.float64)
    want = np.exp2(t.astype(np.float64))
    rel = np.abs(got - want) / want
    assert float(rel.max()) <= 2.0 ** -21, float(np.log2(rel.max()))


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


@pytest.mark.parametrize("kind", [0, 1], ids=["i8", "e4m3"])
def test_mma_loop_runs(kind):
    sink = torch.zeros(149, dtype=torch.int32, device="cuda")
    binding.debug_mma_loop(148, 64, sink, kind)
    torch.cuda.synchronize()
    assert int(sink[148]) == 0

"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the CPU oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from quantized_attention_subtract_b200 import binding
from quantized_attention_subtract_b200.workloads import Workload, generate

# Output tolerances of the GPU path against the oracle (the plain online
# softmax of the quantised method): max |diff| <= 2e-2 and cosine similarity
# >= 0.9999.  Against exact fp64 attention the quantisation itself costs
# ~3.7% relative L1 on iid inputs: FP8 P and FP8 V each contribute the e4m3
# rms rounding error of ~2.65% (pinned in the oracle's CPU tests), INT8 Q K^T
# ~1%; the bound used is 0.06 relative L1 and cosine >= 0.998.
MIRROR_MAX_ABS = 2e-2
MIRROR_COS = 0.9999
EXACT_REL_L1 = 0.06
EXACT_COS = 0.998


def oracle_problem(w: Workload) -> oracle.Problem:
    return oracle.Problem(B=w.B, Hq=w.Hq, Hkv=w.Hkv, Nq=w.Nq, Nkv=w.Nkv, D=w.D, layout=w.layout,
                          dtype=w.dtype, is_causal=w.is_causal, smooth_k=w.smooth_k,
                          smooth_q=w.smooth_q, smooth_v=w.smooth_v, qk_bits=w.qk_bits)


def to_device(bits: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device)
    return t.view(torch.float16 if dtype == "fp16" else torch.bfloat16)


class DeviceRun:
    """Inputs on the device, the output, the workspace and its views."""

    def __init__(self, w: Workload, q, k, v, run_attention: bool = True):
        self.w = w
        self.q, self.k, self.v = (to_device(x, w.dtype) for x in (q, k, v))
        self.out = torch.empty_like(self.q)
        self.p = binding.make_params(self.q, self.k, self.v, self.out, w.layout, w.is_causal, None,
                                     w.smooth_k, w.smooth_q, w.smooth_v, qk_bits=w.qk_bits)
        self.ws = binding.alloc_workspace(self.p, self.q.device)
        if run_attention:
            binding.attn_fwd(self.p, self.q.device)
        else:
            binding.quantize(self.p, self.q.device)
        torch.cuda.synchronize()
        assert binding.device_status(self.p) == 0
        self.views = binding.workspace_views(self.p, self.ws)

    def out_f64(self) -> np.ndarray:
        return self.out.double().cpu().numpy()


def run_both(w: Workload, seed=None):
    q, k, v = generate(w, seed)
    pr = oracle_problem(w)
    pre = oracle.prepass(pr, q, k, v)
    g = DeviceRun(w, q, k, v)
    return q, k, v, pr, pre, g


def assert_prepass_bit_exact(w: Workload, pre: dict, g: DeviceRun):
    V = {k: (v.cpu().numpy() if isinstance(v, torch.Tensor) else v) for k, v in g.views.items()}
    D, Nq, Nkv = w.D, w.Nq, w.Nkv
    q8 = V["q8"]
    assert np.array_equal(q8[:, :, :Nq, :D], pre["q8"]), "q8"
    assert not q8[:, :, Nq:].any() and not q8[:, :, :, D:].any(), "q8 padding"
    k8 = V["k8"]
    assert np.array_equal(k8[:, :, :Nkv, :D], pre["k8"]), "k8"
    assert not k8[:, :, Nkv:].any() and not k8[:, :, :, D:].any(), "k8 padding"
    v8 = V["v8t"].transpose(0, 1, 3, 2)
    assert np.array_equal(v8[:, :, :Nkv], pre["v8"]), "v8"
    assert not v8[:, :, Nkv:].any(), "v8 padding"
    assert np.array_equal(V["q_scale"][:, :, :Nq], pre["q_scale"]), "q_scale"
    assert not V["q_scale"][:, :, Nq:].any(), "q_scale padding"
    nkb = pre["k_scale"].shape[-1]
    assert np.array_equal(V["k_scale"][:, :, :nkb], pre["k_scale"]), "k_scale"
    assert np.array_equal(V["v_scale"], pre["v_scale"]), "v_scale"
    if w.smooth_k:
        assert np.array_equal(V["mean_k"], pre["mean_k"]), "mean_k"
    if w.smooth_v:
        assert np.array_equal(V["mean_v"], pre["mean_v"]), "mean_v"
    if w.smooth_q:
        assert np.array_equal(V["mq"], pre["mq"]), "mq"


def sample_tiles(pr: oracle.Problem, n: int, seed: int = 0) -> np.ndarray:
    """Query tiles to compare at full size: first, last (ragged), and random ones."""
    rng = np.random.default_rng(seed)
    t = [(0, 0, 0), (pr.B - 1, pr.Hq - 1, pr.nqb - 1)]
    while len(t) < n:
        t.append((int(rng.integers(pr.B)), int(rng.integers(pr.Hq)), int(rng.integers(pr.nqb))))
    return np.array(t, np.int32)


def valid_rows(pr: oracle.Problem, tiles) -> np.ndarray:
    m = np.zeros((len(tiles), 128), bool)
    for n, (_, _, qt) in enumerate(np.asarray(tiles).reshape(-1, 3)):
        m[n, : max(0, min(128, pr.Nq - qt * 128))] = True
    return m


def half_ulp(x: np.ndarray, dtype: str) -> np.ndarray:
    """Half a unit in the last place of the 16-bit output type at |x|: the
    largest error of the final round-to-nearest store (bf16 keeps 8
    significant bits, fp16 11; fp16 subnormals have a fixed 2^-24 step)."""
    _, e = np.frexp(np.abs(x))          # |x| = f * 2^e, f in [0.5, 1)
    bits = 8 if dtype == "bf16" else 11
    h = np.ldexp(1.0, e - bits - 1)
    if dtype == "fp16":
        h = np.maximum(h, 2.0 ** -25)
    return h


def compare_output(pr: oracle.Problem, pre: dict, q, k, v, g: DeviceRun, tiles, exact: bool = True):
    """GPU output vs the mirror (and vs exact fp64 attention) on `tiles`.

    max_abs_excess is max(|gpu - mirror| - unc - half_ulp): the part of the
    difference explained neither by FP8 codes of P that the exp2 rounding
    leaves ambiguous (both neighbouring codes valid; the oracle's unc output)
    nor by the final rounding of the output to its 16-bit type."""
    mirror, unc = oracle.attention_tiles(pr, pre, tiles, with_uncertainty=True)
    got = oracle.tile_rows(pr, tiles, g.out_f64())
    rows = valid_rows(pr, tiles)
    a, m, u = got[rows], mirror[rows], unc[rows]
    d = np.abs(a - m)
    hu = half_ulp(np.maximum(np.abs(a), np.abs(m)), pr.dtype)
    res = dict(max_abs=float(d.max()), max_abs_excess=float(np.max(d - u - hu)),
               ambiguous_outputs=int((u > 0).sum()),
               cos=float((a * m).sum() / np.linalg.norm(a) / np.linalg.norm(m)))
    if exact:
        e = oracle.exact_attention_tiles(pr, q, k, v, tiles)[rows]
        res["rel_l1_exact"] = float(np.abs(a - e).sum() / np.abs(e).sum())
        res["cos_exact"] = float((a * e).sum() / np.linalg.norm(a) / np.linalg.norm(e))
        res["mirror_rel_l1_exact"] = float(np.abs(m - e).sum() / np.abs(e).sum())
        res["mirror_cos_exact"] = float((m * e).sum() / np.linalg.norm(m) / np.linalg.norm(e))
    return res

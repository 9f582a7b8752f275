"""Seeded synthetic inputs for the quantized attention forward pass.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic, so both the CPU oracle and the CUDA path can be fed from
it.  Every tensor is drawn in the logical order [B, H, N, D] with numpy's
PCG64 generator and then laid out as HND ([B, H, N, D]) or NHD ([B, N, H, D]),
so the same seed gives the same logical tensors in either layout.

The five named workloads stand in for the model shapes the SageAttention pages
benchmark (language models, video and image generators); no public dataset is
involved.  Value recipes (standard deviations, not variances):

  mha_n256_d64_fp16            B1 H2 N256 D64 fp16 HND; Q,K,V ~ N(0,1);
                               K += per-(b,h,channel) offset ~ N(0, 3)
  mha_n4096_d128_bf16          B4 H32 N4096 D128 bf16 HND; N(0,1); 4 outlier
                               channels per (b,h) scaled x20 in Q, K and V;
                               K offset ~ N(0, 5)
  dit_n17776_d64_bf16_nhd      B2 H48 N17776 D64 bf16 NHD; Q,K ~ N(0,1),
                               K offset ~ N(0, 5); V ~ N(0,1)
  gqa_causal_n32768_d128_bf16  B1 Hq32 Hkv8 N32768 D128 bf16 HND causal;
                               N(0,1); K offset ~ N(0, 5); each token row of
                               Q, K, V independently scaled x10 with prob 2%
  gqa_cross_nq2048_nkv8192_d96_fp16
                               B8 Hq16 Hkv4 Nq2048 Nkv8192 D96 fp16 HND;
                               N(0,1); K offset ~ N(0, 5); run with smooth_k
                               on and off
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nkv: int
    D: int
    layout: str = "HND"
    dtype: str = "bf16"
    is_causal: bool = False
    smooth_k: bool = True
    smooth_q: bool = False
    smooth_v: bool = False
    k_offset_sigma: float = 0.0
    outlier_channels: int = 0
    outlier_scale: float = 1.0
    token_outlier_prob: float = 0.0
    token_outlier_scale: float = 1.0
    seed: int = 0
    qk_bits: int = 8          # bits of the Q and K codes the pass is run with (8 or 4)

    @property
    def ops(self) -> float:
        """Attention operations 4*B*Hq*Nq*Nkv*D, halved for causal."""
        n = 4.0 * self.B * self.Hq * self.Nq * self.Nkv * self.D
        return n / 2 if self.is_causal else n

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("mha_n256_d64_fp16", 1, 2, 2, 256, 256, 64, "HND", "fp16", k_offset_sigma=3.0),
        Workload("mha_n4096_d128_bf16", 4, 32, 32, 4096, 4096, 128, "HND", "bf16",
                 k_offset_sigma=5.0, outlier_channels=4, outlier_scale=20.0),
        Workload("dit_n17776_d64_bf16_nhd", 2, 48, 48, 17776, 17776, 64, "NHD", "bf16",
                 k_offset_sigma=5.0),
        Workload("gqa_causal_n32768_d128_bf16", 1, 32, 8, 32768, 32768, 128, "HND", "bf16",
                 is_causal=True, k_offset_sigma=5.0, token_outlier_prob=0.02,
                 token_outlier_scale=10.0),
        Workload("gqa_cross_nq2048_nkv8192_d96_fp16", 8, 16, 4, 2048, 8192, 96, "HND", "fp16",
                 k_offset_sigma=5.0),
    ]
}


def _to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 -> raw 16-bit patterns (round-half-even) of fp16 or bf16."""
    if dtype == "fp16":
        return x.astype(np.float16).view(np.uint16)
    import torch
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).view(torch.uint16).numpy()


def _layout(x: np.ndarray, layout: str) -> np.ndarray:
    return np.ascontiguousarray(x if layout == "HND" else x.transpose(0, 2, 1, 3))


def generate(w: Workload, seed: int | None = None):
    """Return (q, k, v) as uint16 bit patterns in w.layout, drawn from the seed."""
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    q = rng.standard_normal((w.B, w.Hq, w.Nq, w.D), dtype=np.float32)
    k = rng.standard_normal((w.B, w.Hkv, w.Nkv, w.D), dtype=np.float32)
    v = rng.standard_normal((w.B, w.Hkv, w.Nkv, w.D), dtype=np.float32)
    if w.outlier_channels:
        assert w.Hq == w.Hkv, "channel outliers are drawn per (b, head) of an MHA problem"
        for b in range(w.B):
            for h in range(w.Hq):
                ch = rng.choice(w.D, w.outlier_channels, replace=False)
                q[b, h, :, ch] *= w.outlier_scale
                k[b, h, :, ch] *= w.outlier_scale
                v[b, h, :, ch] *= w.outlier_scale
    if w.token_outlier_prob > 0:
        for x in (q, k, v):
            sel = rng.random(x.shape[:3]) < w.token_outlier_prob
            x[sel] *= w.token_outlier_scale
    if w.k_offset_sigma > 0:
        off = rng.standard_normal((w.B, w.Hkv, 1, w.D), dtype=np.float32) * np.float32(w.k_offset_sigma)
        k += off
    return (_to_bits(_layout(q, w.layout), w.dtype), _to_bits(_layout(k, w.layout), w.dtype),
            _to_bits(_layout(v, w.layout), w.dtype))


def random_problem(B, Hq, Hkv, Nq, Nkv, D, layout="HND", dtype="fp16", seed=0,
                   k_offset_sigma=3.0, **flags) -> Workload:
    """A small ad-hoc workload (tests)."""
    return Workload(f"adhoc_{B}_{Hq}_{Hkv}_{Nq}_{Nkv}_{D}", B, Hq, Hkv, Nq, Nkv, D, layout, dtype,
                    k_offset_sigma=k_offset_sigma, seed=seed, **flags)


def generate_varlen(Hq: int, Hkv: int, D: int, lens_q, lens_kv, dtype: str = "fp16", seed: int = 0,
                    k_offset_sigma: float = 3.0):
    """A packed variable-length batch: returns (cu_q, cu_kv, q, k, v) with
    q [sum(lens_q), Hq, D] and k, v [sum(lens_kv), Hkv, D] as uint16 bit
    patterns (N(0,1); each sequence's K gets its own per-(head, channel)
    offset N(0, k_offset_sigma)), and the int32 offsets."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens_q, lens_kv = np.asarray(lens_q, np.int64), np.asarray(lens_kv, np.int64)
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_kv = np.concatenate([[0], np.cumsum(lens_kv)]).astype(np.int32)
    q = rng.standard_normal((int(cu_q[-1]), Hq, D), dtype=np.float32)
    k = rng.standard_normal((int(cu_kv[-1]), Hkv, D), dtype=np.float32)
    v = rng.standard_normal((int(cu_kv[-1]), Hkv, D), dtype=np.float32)
    if k_offset_sigma > 0:
        for b in range(len(lens_kv)):
            off = rng.standard_normal((1, Hkv, D), dtype=np.float32) * np.float32(k_offset_sigma)
            k[cu_kv[b]:cu_kv[b + 1]] += off
    return cu_q, cu_kv, _to_bits(q, dtype), _to_bits(k, dtype), _to_bits(v, dtype)

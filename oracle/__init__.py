"""CPU oracle for the SageAttention quantized attention forward pass.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow reference the CUDA
path is checked against.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it; the product package never
does, and the two share no code.

The arithmetic lives in ``sage_oracle.c`` (plain C, fp64 except for the fp32
steps whose result is an integer code); this module only builds it with gcc
and marshals numpy arrays.  See the header of ``sage_oracle.c`` for the
passages each step follows and the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sage_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "liboracle.so")

QTILE = 128   # query rows per output tile
QMBLK = 128   # query smoothing-mean block (tokens)
KBLK = 32     # key quantisation block (tokens)
KVT = 128     # keys per online-softmax tile

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile sage_oracle.c with gcc (OpenMP, no FMA contraction)."""
    if not force and os.path.exists(_SO) and os.path.getmtime(_SO) >= os.path.getmtime(_SRC):
        return _SO
    os.makedirs(_BUILD, exist_ok=True)
    tmp = _SO + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _SO)
    return _SO


class _Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("B", "Hq", "Hkv", "Nq", "Nkv", "D", "layout", "dtype",
                 "is_causal", "smooth_k", "smooth_q", "smooth_v")] + [("sm_scale", ctypes.c_float),
                                                                      ("qk_bits", ctypes.c_int)]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.POINTER(_Params)
            vp = ctypes.c_void_p
            lib.oracle_prepass.argtypes = [P] + [vp] * 15
            lib.oracle_attention_tiles.argtypes = [P] + [vp] * 11 + [ctypes.c_int, ctypes.c_int, vp, vp, vp]
            lib.oracle_exact_attention_tiles.argtypes = [P, vp, vp, vp, ctypes.c_int, vp, vp]
            lib.oracle_round_output.argtypes = [P, vp, vp, ctypes.c_int64]
            lib.oracle_e4m3_encode_array.argtypes = [vp, vp, ctypes.c_int64]
            lib.oracle_e4m3_encode_f32_array.argtypes = [vp, vp, ctypes.c_int64]
            lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_decode.restype = ctypes.c_double
            lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
            lib.oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_f16_to_double.restype = ctypes.c_double
            lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_bf16_to_double.restype = ctypes.c_double
            lib.oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


@dataclass
class Problem:
    """Shapes and flags of one call (the oracle's view of sageattn's arguments)."""
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nkv: int
    D: int
    layout: str = "HND"      # "HND" -> [B,H,N,D]; "NHD" -> [B,N,H,D]
    dtype: str = "fp16"      # "fp16" | "bf16"
    is_causal: bool = False
    smooth_k: bool = True
    smooth_q: bool = False
    smooth_v: bool = False
    sm_scale: float | None = None
    qk_bits: int = 8         # 8: INT8 Q/K codes in [-127, 127]; 4: INT4 codes in [-7, 7]

    def resolved_sm_scale(self) -> np.float32:
        if self.sm_scale is not None and self.sm_scale > 0:
            return np.float32(self.sm_scale)
        return np.float32(1.0) / np.sqrt(np.float32(self.D))

    def _c(self) -> _Params:
        return _Params(self.B, self.Hq, self.Hkv, self.Nq, self.Nkv, self.D,
                       0 if self.layout == "HND" else 1, 0 if self.dtype == "fp16" else 1,
                       int(self.is_causal), int(self.smooth_k), int(self.smooth_q),
                       int(self.smooth_v), float(self.resolved_sm_scale()), int(self.qk_bits))

    @property
    def nqb(self) -> int:
        """Query tiles of 128 rows (the output tiling)."""
        return (self.Nq + QTILE - 1) // QTILE

    @property
    def nmb(self) -> int:
        """Query smoothing-mean blocks of 128 tokens."""
        return (self.Nq + QMBLK - 1) // QMBLK

    @property
    def nkb(self) -> int:
        return (self.Nkv + KBLK - 1) // KBLK


def _bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, "inputs are passed as raw 16-bit patterns"
    return x


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def prepass(pr: Problem, q: np.ndarray, k: np.ndarray, v: np.ndarray,
            keep_fp32: bool = False) -> dict:
    """Smoothing + quantisation of Q, K, V (all heads). Inputs: uint16 bit patterns.

    q_scale holds one scale per query token, k_scale one per 32 keys.  With
    keep_fp32 the smoothed fp32 inputs Q' (qp) and V' (vp) are returned too
    (the unquantised operands of the error decomposition)."""
    lib = _load()
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, Hq, Hkv, Nq, Nkv, D = pr.B, pr.Hq, pr.Hkv, pr.Nq, pr.Nkv, pr.D
    out = dict(
        mean_k=np.zeros((B, Hkv, D), np.float32),
        kp=np.zeros((B, Hkv, Nkv, D), np.float32),
        k8=np.zeros((B, Hkv, Nkv, D), np.int8),
        k_scale=np.zeros((B, Hkv, pr.nkb), np.float32),
        mq=np.zeros((B, Hq, pr.nmb, D), np.float32),
        q8=np.zeros((B, Hq, Nq, D), np.int8),
        q_scale=np.zeros((B, Hq, Nq), np.float32),
        mean_v=np.zeros((B, Hkv, D), np.float32),
        v8=np.zeros((B, Hkv, Nkv, D), np.uint8),
        v_scale=np.zeros((B, Hkv, D), np.float32),
    )
    if keep_fp32:
        out["qp"] = np.zeros((B, Hq, Nq, D), np.float32)
        out["vp"] = np.zeros((B, Hkv, Nkv, D), np.float32)
    c = pr._c()
    lib.oracle_prepass(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v),
                       *[_ptr(out[n]) for n in ("mean_k", "kp", "k8", "k_scale", "mq", "q8",
                                                "q_scale", "mean_v", "v8", "v_scale")],
                       _ptr(out["qp"]) if keep_fp32 else None, _ptr(out["vp"]) if keep_fp32 else None)
    return out


def all_tiles(pr: Problem) -> np.ndarray:
    return np.array([(b, h, t) for b in range(pr.B) for h in range(pr.Hq) for t in range(pr.nqb)],
                    np.int32).reshape(-1, 3)


KEEP_P, KEEP_V, KEEP_QK = 1, 2, 4


def attention_tiles(pr: Problem, pre: dict, tiles, with_uncertainty: bool = False,
                    exact_mask: int = 0):
    """The tiled quantised attention (the plain online softmax) for
    (b, h, q_tile) triples.

    Returns fp64 [n_tiles, 128, D] (rows past Nq are zero); with
    `with_uncertainty`, also the per-element bound of how far an fp32
    implementation may differ because an FP8 code of P sits within its
    rounding band of an e4m3 midpoint (see sage_oracle.c).  exact_mask
    (KEEP_P | KEEP_V | KEEP_QK) leaves those steps unquantised, for the error
    decomposition; KEEP_V and KEEP_QK need a pre-pass run with keep_fp32.
    """
    lib = _load()
    tiles = np.ascontiguousarray(np.asarray(tiles, np.int32).reshape(-1, 3))
    out = np.zeros((len(tiles), QTILE, pr.D), np.float64)
    unc = np.zeros_like(out) if with_uncertainty else None
    if exact_mask & (KEEP_V | KEEP_QK):
        assert "qp" in pre and "vp" in pre, "run prepass(..., keep_fp32=True)"
    c = pr._c()
    names = ("q8", "q_scale", "k8", "k_scale", "v8", "v_scale", "mean_v", "mq", "kp")
    lib.oracle_attention_tiles(ctypes.byref(c), *[_ptr(pre[n]) for n in names],
                               _ptr(pre["qp"]) if "qp" in pre else None,
                               _ptr(pre["vp"]) if "vp" in pre else None, int(exact_mask),
                               len(tiles), _ptr(tiles), _ptr(out),
                               _ptr(unc) if unc is not None else None)
    return (out, unc) if with_uncertainty else out


def exact_attention_tiles(pr: Problem, q: np.ndarray, k: np.ndarray, v: np.ndarray, tiles) -> np.ndarray:
    """Exact fp64 softmax attention of the unquantised inputs, same tiling of the output."""
    lib = _load()
    q, k, v = _bits(q), _bits(k), _bits(v)
    tiles = np.ascontiguousarray(np.asarray(tiles, np.int32).reshape(-1, 3))
    out = np.zeros((len(tiles), QTILE, pr.D), np.float64)
    c = pr._c()
    lib.oracle_exact_attention_tiles(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), len(tiles),
                                     _ptr(tiles), _ptr(out))
    return out


def round_output(pr: Problem, x: np.ndarray) -> np.ndarray:
    """fp64 -> 16-bit output dtype bit patterns, round-half-even."""
    lib = _load()
    x = np.ascontiguousarray(x, np.float64)
    bits = np.zeros(x.shape, np.uint16)
    lib.oracle_round_output(ctypes.byref(pr._c()), _ptr(x), _ptr(bits), x.size)
    return bits


def e4m3_encode(x) -> np.ndarray:
    lib = _load()
    x = np.ascontiguousarray(np.asarray(x, np.float64))
    out = np.zeros(x.shape, np.uint8)
    lib.oracle_e4m3_encode_array(_ptr(x), _ptr(out), x.size)
    return out


def e4m3_encode_f32(x) -> np.ndarray:
    lib = _load()
    x = np.ascontiguousarray(np.asarray(x, np.float32))
    out = np.zeros(x.shape, np.uint8)
    lib.oracle_e4m3_encode_f32_array(_ptr(x), _ptr(out), x.size)
    return out


def e4m3_decode_table() -> np.ndarray:
    lib = _load()
    return np.array([lib.oracle_e4m3_decode(c) for c in range(256)], np.float64)


def to_double(pr: Problem, bits: np.ndarray) -> np.ndarray:
    """Decode 16-bit input patterns to fp64 with the oracle's own decoders."""
    lib = _load()
    f = lib.oracle_f16_to_double if pr.dtype == "fp16" else lib.oracle_bf16_to_double
    table = np.array([f(i) for i in range(65536)], np.float64)
    return table[bits]


def tile_rows(pr: Problem, tiles, x: np.ndarray):
    """Gather rows of an [.., D] output in (b, h, q_tile) tiling: returns [n, 128, D]
    (rows past Nq zero).  `x` is a full output in the problem's layout."""
    tiles = np.asarray(tiles, np.int32).reshape(-1, 3)
    out = np.zeros((len(tiles), QTILE, pr.D), x.dtype)
    for n, (b, h, t) in enumerate(tiles):
        i0, i1 = t * QTILE, min(t * QTILE + QTILE, pr.Nq)
        if pr.layout == "HND":
            out[n, : i1 - i0] = x[b, h, i0:i1]
        else:
            out[n, : i1 - i0] = x[b, i0:i1, h]
    return out


def delta_s(pr: Problem, pre: dict, b: int, h: int, qt: int) -> np.ndarray:
    """Q-smoothing correction row dS[j] = mq(b,h,qt) . K'(b,kv(h),j) in fp64
    (qt indexes the 128-token smoothing-mean blocks)."""
    lib = _load()
    lib.oracle_delta_s.argtypes = [ctypes.POINTER(_Params), ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_void_p]
    hk = h // (pr.Hq // pr.Hkv)
    mq = np.ascontiguousarray(pre["mq"][b, h, qt])
    kp = np.ascontiguousarray(pre["kp"][b, hk])
    out = np.zeros(pr.Nkv, np.float64)
    lib.oracle_delta_s(ctypes.byref(pr._c()), _ptr(mq), _ptr(kp), _ptr(out))
    return out


def varlen_attention(Hq: int, Hkv: int, D: int, cu_q, cu_kv, q: np.ndarray, k: np.ndarray,
                     v: np.ndarray, dtype: str = "fp16", is_causal: bool = False,
                     smooth_k: bool = True, smooth_q: bool = False, smooth_v: bool = False,
                     sm_scale: float | None = None, with_uncertainty: bool = False,
                     exact: bool = False, qk_bits: int = 8) -> dict:
    """A variable-length batch of packed sequences (the sageattention package
    page lists batches whose sequences differ in length): sequence b is rows
    cu_q[b] .. cu_q[b+1] of q [total_q, Hq, D] attending to rows
    cu_kv[b] .. cu_kv[b+1] of k, v [total_kv, Hkv, D], and nothing else.
    The pages fix no more than that; the reading taken is that each sequence
    is its own problem -- its own smoothing means, scales and causal mask --
    so this is the single-problem oracle run once per sequence.

    Returns {"out": fp64 [total_q, Hq, D] (the mirror), "pre": [per-sequence
    pre-pass dicts], "problems": [per-sequence Problem]}, plus "unc" and
    "exact" of the output's shape when asked."""
    cu_q, cu_kv = np.asarray(cu_q, np.int64), np.asarray(cu_kv, np.int64)
    total_q = int(cu_q[-1])
    res = {"out": np.zeros((total_q, Hq, D)), "pre": [], "problems": []}
    if with_uncertainty:
        res["unc"] = np.zeros_like(res["out"])
    if exact:
        res["exact"] = np.zeros_like(res["out"])
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_kv[b]), int(cu_kv[b + 1])
        pr = Problem(B=1, Hq=Hq, Hkv=Hkv, Nq=q1 - q0, Nkv=k1 - k0, D=D, layout="NHD", dtype=dtype,
                     is_causal=is_causal, smooth_k=smooth_k, smooth_q=smooth_q, smooth_v=smooth_v,
                     sm_scale=sm_scale, qk_bits=qk_bits)
        res["problems"].append(pr)
        if q1 == q0:
            res["pre"].append(None)
            continue
        qs, ks, vs = (np.ascontiguousarray(x[None]) for x in (q[q0:q1], k[k0:k1], v[k0:k1]))
        pre = prepass(pr, qs, ks, vs)
        res["pre"].append(pre)
        tiles = all_tiles(pr)
        parts = {"out": None, "unc": None, "exact": None}
        if with_uncertainty:
            parts["out"], parts["unc"] = attention_tiles(pr, pre, tiles, with_uncertainty=True)
        else:
            parts["out"] = attention_tiles(pr, pre, tiles)
        if exact:
            parts["exact"] = exact_attention_tiles(pr, qs, ks, vs, tiles)
        for n, (_, h, t) in enumerate(tiles):
            i0, i1 = t * QTILE, min(t * QTILE + QTILE, pr.Nq)
            for name, arr in parts.items():
                if arr is not None:
                    res[name][q0 + i0:q0 + i1, h] = arr[n, :i1 - i0]
    return res

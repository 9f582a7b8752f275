"""Thin ctypes binding of libsage_b200.so (the C ABI in include/sage_b200.h).

Argument marshalling only: every step of the pass runs in the library's CUDA
kernels.  PyTorch supplies device memory (inputs, output, workspace) and the
current stream.  There is no fallback: if the library is missing or the
device is not sm_100, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsage_b200.so")

SAGE_OK = 0
STATUS_NAMES = {0: "SAGE_OK", 1: "SAGE_ERR_INVALID_ARG", 2: "SAGE_ERR_UNSUPPORTED",
                3: "SAGE_ERR_ALIGNMENT", 4: "SAGE_ERR_CUDA", 5: "SAGE_ERR_DEVICE_TIMEOUT",
                6: "SAGE_ERR_WORKSPACE"}

# Every symbol include/sage_b200.h declares.
EXPORTED = ["sage_abi_version", "sage_status_string", "sage_workspace_size", "sage_workspace_view",
            "sage_attn_fwd", "sage_quantize", "sage_attn_quantized", "sage_debug_dump_s",
            "sage_debug_pv", "sage_debug_e4m3", "sage_debug_ex2", "sage_debug_mma_loop",
            "sage_debug_wait_timeout", "sage_get_device_status", "sage_attn_fwd_noalloc",
            "sage_noalloc_device_status", "sage_attn_fwd_prepass", "sage_attn_fwd_attention"]

ABI_VERSION = 5


class SageError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)}")
        self.code = code


class Params(ctypes.Structure):
    """Mirror of sage_attn_params_t."""
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("out", ctypes.c_void_p),
        ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
        ("Nq", ctypes.c_int32), ("Nkv", ctypes.c_int32), ("D", ctypes.c_int32),
        ("q_strides", ctypes.c_int64 * 4), ("k_strides", ctypes.c_int64 * 4),
        ("v_strides", ctypes.c_int64 * 4), ("o_strides", ctypes.c_int64 * 4),
        ("layout", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("is_causal", ctypes.c_int32), ("smooth_k", ctypes.c_int32),
        ("smooth_q", ctypes.c_int32), ("smooth_v", ctypes.c_int32),
        ("sm_scale", ctypes.c_float),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_kv", ctypes.c_void_p),
        ("qk_bits", ctypes.c_int32),
    ]


class WorkspaceView(ctypes.Structure):
    """Mirror of sage_workspace_view_t."""
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("q8", "k8", "v8t", "q_scale", "k_scale", "v_scale", "mean_k", "mean_v", "mq",
                 "dsk", "status")] + [("Dp", ctypes.c_int32), ("Nq_pad", ctypes.c_int32),
                                      ("Nkv_pad", ctypes.c_int32)]


_lock = threading.Lock()
_lib = None


def lib():
    """Load libsage_b200.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"CUDA library missing: {LIB_PATH} (run "
                                   "`python -m quantized_attention_subtract_b200.build`)")
            L = ctypes.CDLL(LIB_PATH)
            P = ctypes.POINTER(Params)
            vp, i32 = ctypes.c_void_p, ctypes.c_int32
            L.sage_abi_version.restype = i32
            L.sage_status_string.restype = ctypes.c_char_p
            L.sage_status_string.argtypes = [ctypes.c_int]
            L.sage_workspace_size.argtypes = [P, ctypes.POINTER(ctypes.c_size_t)]
            L.sage_workspace_view.argtypes = [P, ctypes.POINTER(WorkspaceView)]
            for f in (L.sage_attn_fwd, L.sage_quantize, L.sage_attn_quantized,
                      L.sage_attn_fwd_noalloc, L.sage_attn_fwd_prepass, L.sage_attn_fwd_attention):
                f.argtypes = [P, vp]
            L.sage_debug_dump_s.argtypes = [P, i32, i32, i32, i32, vp, vp]
            L.sage_debug_pv.argtypes = [P, i32, i32, i32, vp, vp, vp]
            L.sage_debug_e4m3.argtypes = [vp, vp, ctypes.c_int64, vp]
            L.sage_debug_ex2.argtypes = [vp, vp, ctypes.c_int64, vp]
            L.sage_debug_mma_loop.argtypes = [i32, i32, i32, vp, vp]
            L.sage_get_device_status.argtypes = [P, ctypes.POINTER(i32)]
            L.sage_noalloc_device_status.argtypes = [P, ctypes.POINTER(i32)]
            L.sage_debug_wait_timeout.argtypes = [vp, vp]
            for name in ("sage_workspace_size", "sage_workspace_view", "sage_attn_fwd",
                         "sage_quantize", "sage_attn_quantized", "sage_debug_dump_s",
                         "sage_debug_pv", "sage_debug_e4m3", "sage_debug_ex2", "sage_debug_mma_loop",
                         "sage_debug_wait_timeout", "sage_get_device_status",
                         "sage_attn_fwd_noalloc", "sage_noalloc_device_status",
                         "sage_attn_fwd_prepass", "sage_attn_fwd_attention"):
                getattr(L, name).restype = ctypes.c_int
            if L.sage_abi_version() != ABI_VERSION:
                raise RuntimeError(f"{LIB_PATH} has ABI version {L.sage_abi_version()}, "
                                   f"this binding expects {ABI_VERSION}: rebuild it")
            _lib = L
    return _lib


def _check(code: int, what: str):
    if code != SAGE_OK:
        raise SageError(code, what)


def _stream(device: torch.device | None = None) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _call(name: str, p, device) -> None:
    """Run entry point `name` on params p and the current stream of `device`,
    with that device current (the library works on the current device)."""
    with torch.cuda.device(device):
        _check(getattr(lib(), name)(ctypes.byref(p), _stream(device)), name)


def _dims(x: torch.Tensor, layout: str):
    if x.dim() != 4:
        raise ValueError("q, k, v must be 4-D")
    if layout == "HND":
        B, H, N, D = x.shape
    elif layout == "NHD":
        B, N, H, D = x.shape
    else:
        raise ValueError(f"tensor_layout must be 'HND' or 'NHD', got {layout!r}")
    return B, H, N, D


def make_params(q, k, v, out=None, tensor_layout="HND", is_causal=False, sm_scale=None,
                smooth_k=True, smooth_q=False, smooth_v=False, workspace=None, qk_bits=8) -> Params:
    """Fill sage_attn_params_t from torch tensors (no copies, strides as given).
    qk_bits: 8 (INT8 Q and K codes) or 4 (INT4 codes in [-7, 7])."""
    B, Hq, Nq, D = _dims(q, tensor_layout)
    Bk, Hkv, Nkv, Dk = _dims(k, tensor_layout)
    if v.shape != k.shape:
        raise ValueError("k and v must have the same shape")
    if (Bk, Dk) != (B, D):
        raise ValueError("q and k disagree on batch or head_dim")
    if q.dtype not in (torch.float16, torch.bfloat16) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share dtype float16 or bfloat16")
    p = Params()
    p.q, p.k, p.v = q.data_ptr(), k.data_ptr(), v.data_ptr()
    p.out = out.data_ptr() if out is not None else None
    p.B, p.Hq, p.Hkv, p.Nq, p.Nkv, p.D = B, Hq, Hkv, Nq, Nkv, D
    for name, t in (("q_strides", q), ("k_strides", k), ("v_strides", v), ("o_strides", out)):
        st = t.stride() if t is not None else (0, 0, 0, 1)
        getattr(p, name)[:] = list(st)
    p.layout = 0 if tensor_layout == "HND" else 1
    p.dtype = 0 if q.dtype == torch.float16 else 1
    p.is_causal, p.smooth_k, p.smooth_q, p.smooth_v = (int(bool(is_causal)), int(bool(smooth_k)),
                                                       int(bool(smooth_q)), int(bool(smooth_v)))
    p.sm_scale = float(sm_scale) if sm_scale is not None else 0.0
    p.qk_bits = int(qk_bits)
    if workspace is not None:
        p.workspace, p.workspace_bytes = workspace.data_ptr(), workspace.numel()
    return p


def _host_offsets(cu) -> np.ndarray:
    """Sequence offsets as a contiguous host int32 array."""
    if isinstance(cu, torch.Tensor):
        cu = cu.detach().to("cpu").numpy()
    a = np.ascontiguousarray(np.asarray(cu), dtype=np.int32)
    if a.ndim != 1 or a.size < 2:
        raise ValueError("cu_seqlens must be 1-D with at least two entries")
    return a


def make_varlen_params(q, k, v, out, cu_seqlens_q, cu_seqlens_kv, max_seqlen_q=None,
                       max_seqlen_kv=None, is_causal=False, sm_scale=None, smooth_k=True,
                       smooth_q=False, smooth_v=False, workspace=None, qk_bits=8) -> Params:
    """sage_attn_params_t for a variable-length batch: q [total_q, Hq, D],
    k, v [total_kv, Hkv, D] (packed sequences), out like q; cu_seqlens_* hold
    B + 1 offsets (host or device integer tensors / arrays, copied to host
    int32)."""
    cq, ck = _host_offsets(cu_seqlens_q), _host_offsets(cu_seqlens_kv)
    if cq.size != ck.size:
        raise ValueError("cu_seqlens_q and cu_seqlens_kv must have the same length")
    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape:
        raise ValueError("packed q, k, v must be [total, heads, head_dim]")
    if q.shape[2] != k.shape[2]:
        raise ValueError("q and k disagree on head_dim")
    if q.dtype not in (torch.float16, torch.bfloat16) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share dtype float16 or bfloat16")
    lq, lk = np.diff(cq), np.diff(ck)
    p = Params()
    p.q, p.k, p.v = q.data_ptr(), k.data_ptr(), v.data_ptr()
    p.out = out.data_ptr() if out is not None else None
    p.B, p.Hq, p.Hkv, p.D = cq.size - 1, q.shape[1], k.shape[1], q.shape[2]
    p.Nq = int(max_seqlen_q) if max_seqlen_q is not None else int(max(lq.max(), 0))
    p.Nkv = int(max_seqlen_kv) if max_seqlen_kv is not None else int(max(lk.max(), 0))
    # NHD order (batch, token, head, channel); the batch stride is unused
    for name, t in (("q_strides", q), ("k_strides", k), ("v_strides", v), ("o_strides", out)):
        st = t.stride() if t is not None else (0, 0, 1)
        getattr(p, name)[:] = [0, st[0], st[1], st[2]]
    p.layout = 1
    p.dtype = 0 if q.dtype == torch.float16 else 1
    p.is_causal, p.smooth_k, p.smooth_q, p.smooth_v = (int(bool(is_causal)), int(bool(smooth_k)),
                                                       int(bool(smooth_q)), int(bool(smooth_v)))
    p.sm_scale = float(sm_scale) if sm_scale is not None else 0.0
    p.qk_bits = int(qk_bits)
    p.cu_seqlens_q, p.cu_seqlens_kv = cq.ctypes.data, ck.ctypes.data
    p._offsets = (cq, ck)  # the arrays must outlive every call made with p
    if workspace is not None:
        p.workspace, p.workspace_bytes = workspace.data_ptr(), workspace.numel()
    return p


def sageattn_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens_q, cu_seqlens_k,
                    max_seqlen_q: int | None = None, max_seqlen_k: int | None = None,
                    is_causal: bool = False, sm_scale: float | None = None, smooth_k: bool = True,
                    smooth_q: bool = False, smooth_v: bool = False, out: torch.Tensor | None = None,
                    workspace: torch.Tensor | None = None, qk_bits: int = 8) -> torch.Tensor:
    """Quantized attention over a variable-length batch of packed sequences on
    the current CUDA stream: q [total_q, Hq, D], k, v [total_kv, Hkv, D] on
    the device; sequence b owns tokens cu_seqlens_q[b] .. cu_seqlens_q[b+1]
    of q (cu_seqlens_k of k, v) and attends only within itself.  Returns out
    shaped like q.  qk_bits as in sageattn."""
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors")
    dev_out = torch.empty_like(q) if out is None else out
    p = make_varlen_params(q, k, v, dev_out, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                           is_causal, sm_scale, smooth_k, smooth_q, smooth_v, qk_bits=qk_bits)
    ws = workspace if workspace is not None else alloc_workspace(p, q.device)
    if workspace is not None:
        p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    attn_fwd(p, q.device)
    return dev_out


def workspace_bytes(p: Params) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().sage_workspace_size(ctypes.byref(p), ctypes.byref(n)), "sage_workspace_size")
    return int(n.value)


def alloc_workspace(p: Params, device) -> torch.Tensor:
    """A workspace of the right size (torch allocations are 512-byte aligned)."""
    ws = torch.empty(workspace_bytes(p), dtype=torch.uint8, device=device)
    p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    return ws


def sageattn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, tensor_layout: str = "HND",
             is_causal: bool = False, sm_scale: float | None = None, smooth_k: bool = True,
             smooth_q: bool = False, smooth_v: bool = False, out: torch.Tensor | None = None,
             workspace: torch.Tensor | None = None, qk_bits: int = 8) -> torch.Tensor:
    """Quantized attention forward: INT8 Q K^T, FP8 P V, on the current CUDA stream.

    q: [B, Hq, Nq, D] ("HND") or [B, Nq, Hq, D] ("NHD"); k, v: same with Hkv, Nkv.
    qk_bits=4 selects the 4-bit variant: INT4 codes of Q and K in [-7, 7] on
    the same blocks (one scale per query token, one per 32 keys), for the
    layers that tolerate it; 8 keeps INT8.
    Host (CPU) tensors are moved to the current device and the result back, in
    chunks of whole (batch, kv-head group) slices so that the host-to-device
    copy of one chunk, the kernels of the previous one and the device-to-host
    copy of the one before overlap; the returned host tensor is complete once
    the current stream has passed this call (pinned host tensors make the
    copies asynchronous).
    """
    if not q.is_cuda:
        return _sageattn_host(q, k, v, tensor_layout, is_causal, sm_scale, smooth_k, smooth_q,
                              smooth_v, out, qk_bits)
    if not (k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be on the same device")
    dev_out = torch.empty_like(q) if out is None else out
    p = make_params(q, k, v, dev_out, tensor_layout, is_causal, sm_scale, smooth_k, smooth_q,
                    smooth_v, qk_bits=qk_bits)
    if workspace is None:
        workspace = alloc_workspace(p, q.device)
    else:
        p.workspace, p.workspace_bytes = workspace.data_ptr(), workspace.numel()
    _call("sage_attn_fwd", p, q.device)
    return dev_out


# Copy/compute pipelining of host-tensor calls: at least this many bytes of
# inputs per chunk, at most this many chunks.
_HOST_CHUNK_MIN_BYTES = 8 << 20
_HOST_MAX_CHUNKS = 16


def _host_chunks(B: int, Hkv: int, group: int, bytes_per_kv_head: int, layout: str = "HND"):
    """Split (batch, kv head) into slices [(b, h0, h1)] of whole kv heads that
    are contiguous in host memory: head ranges of one batch entry for HND, whole
    batch entries for NHD (a head range of an NHD tensor is strided, and a
    strided host-to-device copy goes through a pageable staging copy)."""
    if layout == "NHD":
        return [(b, 0, Hkv) for b in range(B)]
    total = B * Hkv
    n = max(1, min(_HOST_MAX_CHUNKS, total, (total * bytes_per_kv_head) // _HOST_CHUNK_MIN_BYTES))
    per_batch = -(-n // B)                       # chunks per batch entry
    per_b = -(-Hkv // per_batch)                 # kv heads per chunk
    chunks = []
    for b in range(B):
        for h0 in range(0, Hkv, per_b):
            chunks.append((b, h0, min(Hkv, h0 + per_b)))
    return chunks


def _sageattn_host(q, k, v, layout, is_causal, sm_scale, smooth_k, smooth_q, smooth_v, out, qk_bits=8):
    dev = torch.device("cuda", torch.cuda.current_device())
    B, Hq, Nq, D = _dims(q, layout)
    _, Hkv, Nkv, _ = _dims(k, layout)
    group = Hq // Hkv if Hkv else 1
    res = out if out is not None else torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    hq_axis = 1 if layout == "HND" else 2
    # whole-problem device buffers; each chunk is a (batch, head-range) view
    qd, kd, vd = (torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (q, k, v))
    od = torch.empty(q.shape, dtype=q.dtype, device=dev)
    per_kv = (k.element_size() * Nkv * D * 2 + q.element_size() * group * Nq * D * 2)
    chunks = _host_chunks(B, Hkv, group, per_kv, layout)

    def sl(t, b, h0, h1):
        idx = [slice(b, b + 1), slice(None), slice(None), slice(None)]
        idx[hq_axis] = slice(h0, h1)
        return t[tuple(idx)]

    compute = torch.cuda.current_stream(dev)
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    h2d.wait_stream(compute)
    first = make_params(sl(qd, *chunks[0][:1], chunks[0][1] * group, chunks[0][2] * group),
                        sl(kd, *chunks[0]), sl(vd, *chunks[0]),
                        sl(od, chunks[0][0], chunks[0][1] * group, chunks[0][2] * group),
                        layout, is_causal, sm_scale, smooth_k, smooth_q, smooth_v, qk_bits=qk_bits)
    ws = alloc_workspace(first, dev)
    done_out = None
    for b, h0, h1 in chunks:
        qh, kh, vh = sl(q, b, h0 * group, h1 * group), sl(k, b, h0, h1), sl(v, b, h0, h1)
        qc, kc, vc = sl(qd, b, h0 * group, h1 * group), sl(kd, b, h0, h1), sl(vd, b, h0, h1)
        oc, ohost = sl(od, b, h0 * group, h1 * group), sl(res, b, h0 * group, h1 * group)
        with torch.cuda.stream(h2d):
            qc.copy_(qh, non_blocking=True)
            kc.copy_(kh, non_blocking=True)
            vc.copy_(vh, non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(h2d)
        compute.wait_event(landed)
        p = make_params(qc, kc, vc, oc, layout, is_causal, sm_scale, smooth_k, smooth_q, smooth_v,
                        qk_bits=qk_bits)
        need = workspace_bytes(p)
        if need > ws.numel():
            ws = torch.empty(need, dtype=torch.uint8, device=dev)
        p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
        _call("sage_attn_fwd", p, dev)
        computed = torch.cuda.Event()
        computed.record(compute)
        d2h.wait_event(computed)
        with torch.cuda.stream(d2h):
            ohost.copy_(oc, non_blocking=True)
            done_out = torch.cuda.Event()
            done_out.record(d2h)
    compute.wait_event(done_out)
    # keep the device buffers alive until the queued work has used them
    for t in (qd, kd, vd, od, ws):
        t.record_stream(compute)
    return res


NOALLOC_MAX_WORKSPACE_BYTES = 64 << 20


def attn_fwd_noalloc(p: Params, device) -> None:
    """sage_attn_fwd on the library's own static scratch (p.workspace is
    ignored); for callers that cannot allocate device memory on the call path.
    Calls share that scratch: serialise them."""
    _call("sage_attn_fwd_noalloc", p, device)


def noalloc_device_status(p: Params, device) -> int:
    """Device status word the last attn_fwd_noalloc call with p's shapes left."""
    code = ctypes.c_int32(0)
    with torch.cuda.device(device):
        _check(lib().sage_noalloc_device_status(ctypes.byref(p), ctypes.byref(code)),
               "sage_noalloc_device_status")
    return int(code.value)


def quantize(p: Params, device) -> None:
    _call("sage_quantize", p, device)


def attn_quantized(p: Params, device) -> None:
    _call("sage_attn_quantized", p, device)


def attn_fwd(p: Params, device) -> None:
    _call("sage_attn_fwd", p, device)


def attn_fwd_prepass(p: Params, device) -> None:
    _call("sage_attn_fwd_prepass", p, device)


def attn_fwd_attention(p: Params, device) -> None:
    _call("sage_attn_fwd_attention", p, device)


def workspace_views(p: Params, workspace: torch.Tensor) -> dict:
    """torch views of the quantised tensors inside the workspace."""
    w = WorkspaceView()
    _check(lib().sage_workspace_view(ctypes.byref(p), ctypes.byref(w)), "sage_workspace_view")
    base = workspace.data_ptr()

    def view(addr, n, dtype, shape):
        off = addr - base
        esize = torch.tensor([], dtype=dtype).element_size()
        return workspace[off: off + n * esize].view(dtype).view(*shape)

    B, Hq, Hkv, D = p.B, p.Hq, p.Hkv, p.D
    nqb, nkb = w.Nq_pad // 128, w.Nkv_pad // 32
    out = dict(
        q8=view(w.q8, B * Hq * w.Nq_pad * w.Dp, torch.int8, (B, Hq, w.Nq_pad, w.Dp)),
        k8=view(w.k8, B * Hkv * w.Nkv_pad * w.Dp, torch.int8, (B, Hkv, w.Nkv_pad, w.Dp)),
        v8t=view(w.v8t, B * Hkv * D * w.Nkv_pad, torch.uint8, (B, Hkv, D, w.Nkv_pad)),
        q_scale=view(w.q_scale, B * Hq * w.Nq_pad, torch.float32, (B, Hq, w.Nq_pad)),
        k_scale=view(w.k_scale, B * Hkv * nkb, torch.float32, (B, Hkv, nkb)),
        v_scale=view(w.v_scale, B * Hkv * D, torch.float32, (B, Hkv, D)),
        mean_k=view(w.mean_k, B * Hkv * D, torch.float32, (B, Hkv, D)),
        mean_v=view(w.mean_v, B * Hkv * D, torch.float32, (B, Hkv, D)),
        status=view(w.status, 1, torch.int32, (1,)),
        Dp=w.Dp, Nq_pad=w.Nq_pad, Nkv_pad=w.Nkv_pad,
    )
    if w.mq:
        out["mq"] = view(w.mq, B * Hq * nqb * D, torch.float32, (B, Hq, nqb, D))
        out["dsk"] = view(w.dsk, B * Hq * nqb * w.Nkv_pad, torch.float32, (B, Hq, nqb, w.Nkv_pad))
    return out


def debug_dump_s(p: Params, b: int, h: int, qtile: int, ktile: int, device) -> torch.Tensor:
    """The attention half of the pass in the S-dump build of the attention
    kernel: returns the int32 S tile (qtile, ktile) of (b, h) as its softmax
    warps read it (filled with -1 where the kernel computed no such tile);
    writes p.out too."""
    s = torch.full((128, 128), -1, dtype=torch.int32, device=device)
    with torch.cuda.device(device):
        _check(lib().sage_debug_dump_s(ctypes.byref(p), b, h, qtile, ktile,
                                       ctypes.c_void_p(s.data_ptr()), _stream(device)),
               "sage_debug_dump_s")
    return s


def debug_pv(p: Params, b: int, hkv: int, ktile: int, p8: torch.Tensor, device) -> torch.Tensor:
    assert p8.dtype == torch.uint8 and p8.shape == (128, 128) and p8.is_contiguous()
    o = torch.empty((128, p.D), dtype=torch.float32, device=device)
    _check(lib().sage_debug_pv(ctypes.byref(p), b, hkv, ktile, ctypes.c_void_p(p8.data_ptr()),
                               ctypes.c_void_p(o.data_ptr()), _stream(device)), "sage_debug_pv")
    return o


def debug_e4m3(x: torch.Tensor) -> torch.Tensor:
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(lib().sage_debug_e4m3(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                 x.numel(), _stream(x.device)), "sage_debug_e4m3")
    return out


def debug_mma_loop(ctas: int, iters: int, sink: torch.Tensor, kind: int = 0) -> None:
    """Back-to-back 8-bit MMAs (kind 0 INT8, kind 1 FP8 e4m3); sink: int32
    device tensor with at least ctas + 1 entries (the last one is a status word)."""
    assert sink.dtype == torch.int32 and sink.numel() >= ctas + 1
    _check(lib().sage_debug_mma_loop(ctas, iters, kind, ctypes.c_void_p(sink.data_ptr()),
                                     _stream(sink.device)), "sage_debug_mma_loop")


def debug_ex2(x: torch.Tensor) -> torch.Tensor:
    """The attention kernel's exp2 applied to a float32 device tensor."""
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()
    out = torch.empty_like(x)
    _check(lib().sage_debug_ex2(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                x.numel(), _stream(x.device)), "sage_debug_ex2")
    return out


def debug_wait_timeout(status: torch.Tensor) -> None:
    """Run a bounded wait that nothing completes; status[0] becomes SAGE_ERR_DEVICE_TIMEOUT."""
    assert status.dtype == torch.int32 and status.is_cuda
    _check(lib().sage_debug_wait_timeout(ctypes.c_void_p(status.data_ptr()), _stream(status.device)),
           "sage_debug_wait_timeout")


def device_status(p: Params) -> int:
    code = ctypes.c_int32(0)
    _check(lib().sage_get_device_status(ctypes.byref(p), ctypes.byref(code)),
           "sage_get_device_status")
    return int(code.value)

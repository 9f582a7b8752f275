"""The C ABI library: loads without a GPU, exports every declared symbol, and
rejects out-of-contract arguments before touching the device."""
import ctypes
import os
import re

import pytest

from quantized_attention_subtract_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sage_b200.h")
GOLDEN = os.path.join(ROOT, "tests", "golden", "api_contract.txt")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^[a-z_0-9 \*]+?\b(sage_[a-z_0-9]+)\(", text, re.M)))


def test_library_exports_every_declared_symbol():
    L = binding.lib()
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert sorted(binding.EXPORTED) == names
    assert L.sage_abi_version() == binding.ABI_VERSION == 5


def test_status_strings():
    L = binding.lib()
    for code, name in binding.STATUS_NAMES.items():
        assert L.sage_status_string(code).decode() == name


def _params(**kw):
    p = binding.Params()
    d = dict(B=1, Hq=2, Hkv=2, Nq=256, Nkv=256, D=64, layout=0, dtype=0, is_causal=0, smooth_k=1)
    d.update(kw)
    for k, v in d.items():
        setattr(p, k, v)
    for name in ("q_strides", "k_strides", "v_strides", "o_strides"):
        getattr(p, name)[:] = [d["Hq"] * d["Nq"] * d["D"], d["Nq"] * d["D"], d["D"], 1]
    return p


def _ws_size(p):
    n = ctypes.c_size_t(0)
    return binding.lib().sage_workspace_size(ctypes.byref(p), ctypes.byref(n)), n.value


@pytest.mark.parametrize("bits,ok", [(0, True), (8, True), (4, True), (1, False), (5, False),
                                     (16, False), (-4, False)])
def test_qk_bits_values(bits, ok):
    st, n = _ws_size(_params(qk_bits=bits))
    assert (st == 0) == ok
    if ok:
        # the 4-bit codes live in the same buffers: same workspace size
        assert n == _ws_size(_params())[1]


def _contract():
    facts = {}
    for line in open(GOLDEN):
        if line.strip() and not line.startswith("#"):
            key, *vals = line.split()
            facts[key] = vals
    return facts


def test_head_dims_follow_the_pages():
    allowed = {int(x) for x in _contract()["head_dims"]}
    for D in range(16, 257, 16):
        code, _ = _ws_size(_params(D=D))
        assert (code == 0) == (D in allowed), D
    assert _ws_size(_params(D=96))[0] == 0


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=6, Hkv=4), 1), (dict(Nkv=0), 1), (dict(B=0), 1), (dict(Nq=-1), 1),
    (dict(layout=2), 1), (dict(dtype=5), 2), (dict(is_causal=2), 1), (dict(D=80), 2),
])
def test_bad_shapes_rejected(kw, code):
    assert _ws_size(_params(**kw))[0] == code


def test_workspace_size_grows_with_smooth_q():
    base = _ws_size(_params())[1]
    withq = _ws_size(_params(smooth_q=1))[1]
    assert withq > base > 0


def _fwd(p):
    return binding.lib().sage_attn_fwd(ctypes.byref(p), None)


def test_argument_errors_before_any_device_work():
    p = _params()
    fake = 1 << 40  # never dereferenced: validation fails first
    p.q = p.k = p.v = p.out = fake
    p.workspace, p.workspace_bytes = fake, _ws_size(p)[1]
    bad = _params()
    bad.q = bad.k = bad.v = bad.out = fake + 8  # not 16-byte aligned
    bad.workspace, bad.workspace_bytes = fake, p.workspace_bytes
    assert _fwd(bad) == 3
    p2 = _params()
    p2.q = p2.k = p2.v = p2.out = fake
    p2.q_strides[2] = 68  # token stride not a multiple of 8 elements
    p2.workspace, p2.workspace_bytes = fake, p.workspace_bytes
    assert _fwd(p2) == 3
    p3 = _params()
    p3.q = p3.k = p3.v = p3.out = fake
    p3.workspace, p3.workspace_bytes = fake, p.workspace_bytes - 1
    assert _fwd(p3) == 6
    p4 = _params()
    p4.q = p4.k = p4.v = p4.out = fake
    p4.workspace, p4.workspace_bytes = fake + 128, p.workspace_bytes
    assert _fwd(p4) == 6
    p5 = _params()
    p5.q = None
    p5.workspace, p5.workspace_bytes = fake, p.workspace_bytes
    assert _fwd(p5) == 1


def test_binding_raises_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(RuntimeError, match="CUDA library missing"):
        binding.lib()


def test_python_mirrors_match_the_c_structs(tmp_path):
    """binding.Params / WorkspaceView have the size and field offsets that a C
    compiler gives sage_attn_params_t / sage_workspace_view_t from the header."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    hdr = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    mirrors = (("sage_attn_params_t", binding.Params), ("sage_workspace_view_t", binding.WorkspaceView))
    lines = ['#include <stdio.h>', '#include "sage_b200.h"', "int main(void) {"]
    for cname, py in mirrors:
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for field, _ in py._fields_:
            lines.append(f'  printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", hdr, str(src), "-o", str(exe)], check=True)
    got = dict(l.rsplit(" ", 1) for l in subprocess.run([str(exe)], check=True, capture_output=True,
                                                          text=True).stdout.splitlines())
    for cname, py in mirrors:
        assert int(got[f"{cname} size"]) == ctypes.sizeof(py), cname
        for field, _ in py._fields_:
            assert int(got[f"{cname} {field}"]) == getattr(py, field).offset, (cname, field)


def _varlen_params(cu_q, cu_kv, **kw):
    """Batched-shape params turned into a variable-length batch with host
    offset arrays (kept alive on the returned object)."""
    import numpy as np
    cq, ck = np.asarray(cu_q, np.int32), np.asarray(cu_kv, np.int32)
    p = _params(B=len(cq) - 1, **kw)
    p.cu_seqlens_q, p.cu_seqlens_kv = cq.ctypes.data, ck.ctypes.data
    p._keep = (cq, ck)
    fake = 1 << 40
    p.q = p.k = p.v = p.out = fake
    p.workspace = fake
    return p


@pytest.mark.parametrize("cu_q,cu_kv,ok", [
    ([0, 100, 256], [0, 200, 256], True),
    ([0, 0, 256], [0, 0, 256], True),         # a sequence without queries needs no keys
    ([1, 100, 256], [0, 200, 256], False),    # must start at 0
    ([0, 200, 100], [0, 100, 200], False),    # decreasing
    ([0, 100, 400], [0, 100, 200], False),    # longer than Nq = 256
    ([0, 100, 200], [0, 0, 200], False),      # queries without keys
])
def test_varlen_offsets_checked_before_any_device_work(cu_q, cu_kv, ok):
    p = _varlen_params(cu_q, cu_kv)
    code, n = _ws_size(p)
    assert code == 0
    # one byte short: valid offsets get as far as the workspace check (and no
    # further, so nothing is launched on any machine); invalid ones stop first
    p.workspace_bytes = n - 1
    assert _fwd(p) == (6 if ok else 1)


def test_varlen_needs_both_offset_arrays():
    p = _varlen_params([0, 100, 256], [0, 200, 256])
    p.cu_seqlens_kv = None
    p.workspace_bytes = _ws_size(p)[1] - 1
    assert _fwd(p) == 1


def test_varlen_workspace_holds_the_offsets():
    batched = _params(B=2)
    _, n0 = _ws_size(batched)
    _, n1 = _ws_size(_varlen_params([0, 100, 256], [0, 200, 256]))
    assert n1 > n0


@pytest.mark.parametrize("layout,B,Hkv,group,N", [("HND", 4, 32, 1, 4096), ("HND", 1, 8, 4, 32768),
                                                   ("HND", 2, 3, 2, 64), ("NHD", 2, 48, 1, 17776),
                                                   ("NHD", 1, 4, 4, 100)])
def test_host_chunks_cover_every_head_once_in_contiguous_slices(layout, B, Hkv, group, N):
    """Host-tensor calls are pipelined over chunks of whole kv heads; every
    (batch, kv head) is in exactly one chunk, and each chunk's slice of a
    dense host tensor is contiguous (a strided slice would be copied through
    pageable staging memory)."""
    import torch
    D = 64
    per_kv = 2 * N * D * 2 + 2 * group * N * D * 2
    chunks = binding._host_chunks(B, Hkv, group, per_kv, layout)
    seen = [(b, h) for b, h0, h1 in chunks for h in range(h0, h1)]
    assert sorted(seen) == [(b, h) for b in range(B) for h in range(Hkv)]
    shape = (B, Hkv * group, N, D) if layout == "HND" else (B, N, Hkv * group, D)
    q = torch.empty(shape, dtype=torch.float16)
    for b, h0, h1 in chunks:
        if layout == "HND":
            view = q[b:b + 1, h0 * group:h1 * group]
        else:
            view = q[b:b + 1, :, h0 * group:h1 * group]
        assert view.is_contiguous(), (b, h0, h1)


@pytest.mark.parametrize("kw,code", [
    # 32-bit TMA row coordinates and kernel indices: B * H * (N rounded up to 128) < 2^31
    (dict(Hq=2, Hkv=2, Nq=(1 << 30) - 128, Nkv=256), 0),
    (dict(Hq=2, Hkv=2, Nq=(1 << 30) - 127, Nkv=256), 2),
    (dict(Hq=2, Hkv=2, Nq=256, Nkv=(1 << 30) - 128), 0),
    (dict(Hq=2, Hkv=2, Nq=256, Nkv=1 << 30), 2),
    (dict(B=(1 << 17) - 1, Hq=128, Hkv=128, Nq=128, Nkv=128), 0),
    (dict(B=1 << 17, Hq=128, Hkv=128, Nq=128, Nkv=128), 2),
])
def test_size_limits(kw, code):
    """The largest problems the 32-bit indices allow are accepted and one
    128-row tile more is rejected as unsupported, before any device work."""
    assert _ws_size(_params(**kw))[0] == code


@pytest.mark.parametrize("scale", [float("nan"), float("inf"), float("-inf")])
def test_non_finite_sm_scale_rejected(scale):
    p = _params()
    p.sm_scale = scale
    assert _ws_size(p)[0] == 1


def test_binding_passes_qk_bits():
    """The Python builders fill sage_attn_params_t.qk_bits (default 8); the
    library sizes the workspace the same for both code widths."""
    import torch
    q = torch.zeros(1, 2, 256, 64, dtype=torch.float16)
    k = torch.zeros(1, 2, 256, 64, dtype=torch.float16)
    p8 = binding.make_params(q, k, k, q)
    p4 = binding.make_params(q, k, k, q, qk_bits=4)
    assert p8.qk_bits == 8 and p4.qk_bits == 4
    assert binding.workspace_bytes(p8) == binding.workspace_bytes(p4)
    qv = torch.zeros(300, 2, 64, dtype=torch.bfloat16)
    kv = torch.zeros(200, 2, 64, dtype=torch.bfloat16)
    pv = binding.make_varlen_params(qv, kv, kv, qv, [0, 100, 300], [0, 50, 200], qk_bits=4)
    assert pv.qk_bits == 4 and pv.B == 2
    bad = binding.make_params(q, k, k, q, qk_bits=5)
    with pytest.raises(binding.SageError):
        binding.workspace_bytes(bad)

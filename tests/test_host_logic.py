"""Host-side logic of the binding and the benchmark, on CPU.

- Host-tensor calls split (batch, kv head) into chunks that cover every pair
  exactly once, each a contiguous range of one batch entry (HND) or a whole
  batch entry (NHD, where a head range is strided in host memory).
- The clock sampler keeps the samples inside the timed region, reports the
  median SM clock and every active throttle reason.
- The recorded attention DRAM traffic is reported only for the kernel sources
  it was measured on.
- The oracle sample of the reference arm grows with the time it is given.
"""
import os

import pytest

import bench
from quantized_attention_subtract_b200 import binding
from quantized_attention_subtract_b200.workloads import WORKLOADS


@pytest.mark.parametrize("B,Hkv,group,per_kv", [(1, 8, 4, 64 << 20), (4, 32, 1, 4 << 20),
                                                (2, 3, 2, 1 << 30), (8, 4, 4, 1 << 10)])
def test_host_chunks_cover_every_head_once_hnd(B, Hkv, group, per_kv):
    chunks = binding._host_chunks(B, Hkv, group, per_kv, "HND")
    seen = [(b, h) for b, h0, h1 in chunks for h in range(h0, h1)]
    assert sorted(seen) == [(b, h) for b in range(B) for h in range(Hkv)]
    assert all(0 <= h0 < h1 <= Hkv for _, h0, h1 in chunks)
    assert len(chunks) <= max(B, binding._HOST_MAX_CHUNKS)


def test_host_chunks_nhd_are_whole_batch_entries():
    chunks = binding._host_chunks(3, 8, 4, 64 << 20, "NHD")
    assert chunks == [(0, 0, 8), (1, 0, 8), (2, 0, 8)]


def _sampler_with(tmp_path, lines, t0, t1):
    s = bench.ClockSampler(0)
    p = tmp_path / "clocks.csv"
    p.write_text("\n".join(lines) + "\n")
    s.path, s.proc, s.t0, s.t1 = str(p), object(), t0, t1
    return s


def _row(ts, sm, reasons=("Not Active",) * 4):
    from datetime import datetime
    stamp = datetime.fromtimestamp(ts).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return ", ".join([stamp, "0", str(sm), "1965", "700.00", "0x0"] + list(reasons))


def test_clock_sampler_keeps_the_timed_region(tmp_path):
    t0 = 1_800_000_000.0
    lines = [_row(t0 - 5, 300), _row(t0 + 0.2, 1965), _row(t0 + 0.4, 1950),
             _row(t0 + 0.6, 1965, ("Not Active", "Not Active", "Not Active", "Active")),
             _row(t0 + 9, 100)]
    got = _sampler_with(tmp_path, lines, t0, t0 + 1.0).summary()
    assert got["samples"] == 3 and got["window"] == "timed region"
    assert got["sm_mhz"] == 1965.0 and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"]


def test_clock_sampler_falls_back_to_the_whole_run(tmp_path):
    t0 = 1_800_000_000.0
    lines = [_row(t0 - 3, 1965, ("Active", "Not Active", "Not Active", "Not Active")),
             _row(t0 + 3, 1900)]
    got = _sampler_with(tmp_path, lines, t0, t0 + 0.01).summary()
    assert got["samples"] == 2 and got["window"].startswith("whole run")
    assert got["reasons"] == ["hw_slowdown"]


def test_recorded_traffic_follows_the_kernel_sources(monkeypatch, tmp_path):
    import hashlib
    data = b"".join(open(os.path.join(bench.ROOT, "quantized_attention_subtract_b200", "csrc", f), "rb").read()
                    for f in bench.ATTN_SOURCES)
    current = hashlib.sha256(data).hexdigest()[:16]
    for name, rec in bench.ATTN_TRAFFIC.items():
        want = rec["bytes"] if rec["sources_sha256_16"] == current else None
        assert bench._attn_traffic(WORKLOADS[name]) == want
    assert bench._attn_traffic(WORKLOADS["dit_n17776_d64_bf16_nhd"]) is None
    # any change to the hashed sources turns the record off
    csrc = tmp_path / "quantized_attention_subtract_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.ATTN_SOURCES:
        src = os.path.join(bench.ROOT, "quantized_attention_subtract_b200", "csrc", f)
        (csrc / f).write_bytes(open(src, "rb").read() + (b"\n" if f == "common.cuh" else b""))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._attn_traffic(WORKLOADS["gqa_causal_n32768_d128_bf16"]) is None


def test_reference_sample_grows_with_its_time(monkeypatch):
    w = WORKLOADS["gqa_causal_n32768_d128_bf16"]
    # one oracle tile takes 10 ms in this fake
    monkeypatch.setattr(bench, "oracle_sample", lambda w_, h, t: (0.0, 0.01 * 2 * (w_.Hq // w_.Hkv), "", 1))
    # a kv head of this workload is 256 query tiles x 4 query heads = 1024 tiles
    assert bench._sample_size(w, 0.2) == (1, 20 // 4)
    assert bench._sample_size(w, 5.0) == (1, 500 // 4)
    assert bench._sample_size(w, 25.0) == (2, None)
    assert bench._sample_size(w, 1e6) == (w.Hkv, None)

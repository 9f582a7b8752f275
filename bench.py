"""Benchmark of the quantized attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--qk-bits 8|4] [--varlen] [--no-cpu-baseline]

A step is one whole pass (smoothing + quantisation pre-pass, then the
attention kernel) over one batch of the named synthetic workload (default:
causal GQA prefill B1 Hq32 Hkv8 N32768 D128 bf16, the N >= 8K, d = 128 case
the throughput target is stated for), inputs resident in HBM.  The metric
is attention TOPS = 4*B*Hq*Nq*Nkv*D / time (halved for causal), whole job.
Under torchrun (N > 1) every rank runs the same workload on its own GPU
(independent replicas, no collective in the data path: the pass does not
shard across GPUs); the time is the max over ranks.

Reported beside the value: the attention kernel's roofline (tensor-bound,
8-bit peak derived from the measured bf16 GEMM peak x 2, the nominal 8-bit /
16-bit ratio, and beside it the rate of back-to-back tcgen05 8-bit MMAs
measured in the same run), the end-to-end number through the public API with
host buffers, SM clocks sampled during the timed region, and the CPU oracle
timed on a bounded sample (``cpu_baseline``).  ``--impl reference`` times the CPU
oracle itself on the same workload, one bounded sample per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_attention_subtract_b200.workloads import WORKLOADS, Workload, generate  # noqa: E402

METRIC = "attention TOPS (4*B*H*Nq*Nkv*d/s) at N=4K-32K, d=128; % of B200 tensor peak"
DEFAULT_WORKLOAD = "gqa_causal_n32768_d128_bf16"
L2_BYTES = 126 * 1024 * 1024

# DRAM bytes (read + write) per launch of the attention kernel, from one ncu
# capture per workload.  They describe the kernel built from the sources hashed
# here; after any change to those sources the traffic is reported as null until
# it is captured again.
ATTN_TRAFFIC = {     # workload name -> {"sources_sha256_16": ..., "bytes": ...}
    "mha_n4096_d128_bf16": {"sources_sha256_16": "a60e3f7d2388b637", "bytes": 203625728 + 104289024},
    "gqa_causal_n32768_d128_bf16": {"sources_sha256_16": "a60e3f7d2388b637", "bytes": 498916352 + 221931264},
}
ATTN_SOURCES = ["attn_fwd.cu", "ptx.cuh", "common.cuh"]


def _prepass_bytes(w: Workload, qd, kd, vd) -> int:
    """Algorithmic bytes of the pre-pass launches of one step: 2 B read and
    1 B written per element of Q, K and V."""
    return 3 * (qd.numel() + kd.numel() + vd.numel())


def _attn_traffic(w: Workload):
    import hashlib
    csrc = os.path.join(ROOT, "quantized_attention_subtract_b200", "csrc")
    try:
        data = b"".join(open(os.path.join(csrc, f), "rb").read() for f in ATTN_SOURCES)
    except OSError:
        return None
    rec = ATTN_TRAFFIC.get(w.name)
    if rec is None or hashlib.sha256(data).hexdigest()[:16] != rec["sources_sha256_16"]:
        return None
    return rec["bytes"]


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return float(m["bf16_tflops"]), float(m["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 6650.0, "fallback"


def mma_loop_peak(dev, iters: int = 4096):
    """TOPS of back-to-back tcgen05 8-bit MMAs (128x256x32, operands resident
    in shared memory) on one CTA per SM, INT8 and FP8 kinds, timed with CUDA
    events after a warm-up: the attainable 8-bit tensor rate of this GPU."""
    import torch
    from quantized_attention_subtract_b200 import binding
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    sink = torch.zeros(sms + 1, dtype=torch.int32, device=dev)
    out = {}
    for kind, name in ((0, "i8"), (1, "e4m3")):
        binding.debug_mma_loop(sms, 256, sink, kind)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        binding.debug_mma_loop(sms, iters, sink, kind)
        b.record()
        torch.cuda.synchronize(dev)
        assert int(sink[sms]) == 0, "MMA loop status"
        ops = 2.0 * 128 * 256 * 128 * iters * sms   # 4 MMAs of K=32 per iteration
        out[name] = ops / (a.elapsed_time(b) * 1e-3) / 1e12
    return out


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise max of per-rank timings (every rank gets the result); with
    no process group the values come back unchanged."""
    if dist is None:
        return [float(x) for x in values]
    import torch
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def replica_value(world: int, ops_per_replica: float, ms: float) -> float:
    """Whole-job TOPS of `world` independent replicas timed at `ms` (max over ranks)."""
    return world * ops_per_replica / (ms * 1e-3) / 1e12


def _oracle_problem(w: Workload):
    import oracle
    return oracle.Problem(B=w.B, Hq=w.Hq, Hkv=w.Hkv, Nq=w.Nq, Nkv=w.Nkv, D=w.D, layout=w.layout,
                          dtype=w.dtype, is_causal=w.is_causal, smooth_k=w.smooth_k,
                          smooth_q=w.smooth_q, smooth_v=w.smooth_v, qk_bits=w.qk_bits)


def oracle_sample(w: Workload, kv_heads: int, q_tiles: int | None = None):
    """Time the CPU oracle (pre-pass + tiled attention) on the first `kv_heads`
    kv heads of batch 0 with all their query heads, on the first `q_tiles`
    query tiles of each (all when None).  Returns (tops, seconds, description,
    threads)."""
    import oracle
    group = w.Hq // w.Hkv
    sub = w.with_(B=1, Hkv=kv_heads, Hq=kv_heads * group)
    q, k, v = generate(sub)
    pr = _oracle_problem(sub)
    tiles = oracle.all_tiles(pr)
    nt = pr.nqb if q_tiles is None else max(1, min(q_tiles, pr.nqb))
    tiles = tiles[tiles[:, 2] < nt]
    t0 = time.perf_counter()
    pre = oracle.prepass(pr, q, k, v)
    oracle.attention_tiles(pr, pre, tiles)
    dt = time.perf_counter() - t0
    rows = sum(min(128, w.Nq - 128 * int(t)) for t in tiles[:, 2])
    ops = 4.0 * rows * w.Nkv * w.D * (0.5 if w.is_causal else 1.0)
    desc = (f"batch 0, kv heads 0..{kv_heads - 1} ({sub.Hq} query heads, query tiles 0..{nt - 1} "
            f"each) of {w.name}: pre-pass of those heads + tiled quantised attention")
    return ops / dt / 1e12, dt, desc, oracle.num_threads()


def _sample_size(w: Workload, target_s: float):
    """(kv_heads, q_tiles) of batch 0 whose oracle run takes about target_s seconds."""
    try:
        _, dt, _, _ = oracle_sample(w, 1, 2)
        per_tile = dt / (2 * (w.Hq // w.Hkv))
    except Exception:
        per_tile = 0.05
    tiles_total = max(1, int(target_s / max(per_tile, 1e-4)))
    nqb = (w.Nq + 127) // 128
    group = w.Hq // w.Hkv
    per_head = nqb * group
    if tiles_total >= per_head:
        return min(w.Hkv, tiles_total // per_head), None
    return 1, max(1, tiles_total // group)


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason samples; summary() keeps the
    samples whose timestamps fall inside the marked timed region."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(1.0)  # let the sampler start before the timed region
        except Exception:
            self.proc = None

    def mark_begin(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        from datetime import datetime
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            rows.append((ts, parts))
        os.unlink(self.path)
        inside = [p for ts, p in rows if self.t0 is not None and self.t0 - 0.1 <= ts <= self.t1 + 0.1]
        use = inside if inside else [p for _, p in rows]
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        num = lambda s: float(s) if s.replace(".", "", 1).isdigit() else None
        sm = [num(r[2]) for r in use if num(r[2]) is not None]
        mx = [num(r[3]) for r in use if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i in range(4) if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(use),
                "window": "timed region" if inside else "whole run (timed region shorter than one sample)"}


def run_reference(args, w: Workload):
    """The CPU oracle timed as the reference arm (rank 0 only)."""
    world, rank, _ = _dist()
    if rank != 0:
        return
    # each step a bounded sample, so the whole run stays near two minutes
    per_step = min(2.0, 120.0 / max(1, args.steps + args.warmup))
    heads, tiles = _sample_size(w, per_step)
    for _ in range(args.warmup):
        oracle_sample(w, heads, tiles)
    times, tops = [], []
    desc, threads = "", 1
    for _ in range(args.steps):
        t, dt, desc, threads = oracle_sample(w, heads, tiles)
        times.append(dt)
        tops.append(t)
    value = float(np.mean(tops))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * float(np.mean(times)),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "i8xi8->i64 (QK), e4m3xe4m3->f64 (PV)", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "Nkv": w.Nkv,
                   "D": w.D, "layout": w.layout, "causal": w.is_causal, "smooth_k": w.smooth_k,
                   "qk_bits": w.qk_bits},
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, w: Workload):
    import torch
    from quantized_attention_subtract_b200 import binding, sageattn

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
        pg = dist

    q, k, v = generate(w)
    to_dev = lambda x: torch.from_numpy(x.view(np.int16)).to(dev).view(
        torch.float16 if w.dtype == "fp16" else torch.bfloat16)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    out = torch.empty_like(qd)
    p = binding.make_params(qd, kd, vd, out, w.layout, w.is_causal, None, w.smooth_k, w.smooth_q,
                            w.smooth_v, qk_bits=w.qk_bits)
    ws = binding.alloc_workspace(p, dev)
    stream = torch.cuda.current_stream(dev)
    in_bytes = qd.numel() * 2 + kd.numel() * 2 + vd.numel() * 2

    def barrier():
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize(dev)

    # ---- warm-up, then K timed steps of the whole pass
    clk = ClockSampler(local)
    clk.start()
    for _ in range(args.warmup):
        binding.attn_fwd(p, dev)
    barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk.mark_begin()
    start.record(stream)
    for _ in range(args.steps):
        binding.attn_fwd(p, dev)
    end.record(stream)
    barrier()
    clk.mark_end()
    step_ms = start.elapsed_time(end) / args.steps
    # ---- the same pass as its two halves (pre-pass launches, then the
    # attention kernel), with events around each half: the attention kernel
    # (the dominant one) and the pre-pass as they run inside a step
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(args.steps)]
    for a, b, c in evs:
        a.record(stream)
        binding.attn_fwd_prepass(p, dev)
        b.record(stream)
        binding.attn_fwd_attention(p, dev)
        c.record(stream)
    torch.cuda.synchronize(dev)
    pre_ms = float(np.mean([a.elapsed_time(b) for a, b, _ in evs]))
    attn_ms = float(np.mean([b.elapsed_time(c) for _, b, c in evs]))
    clk.stop()
    clocks = clk.summary()
    assert binding.device_status(p) == 0, "device status nonzero"

    # max over ranks
    step_ms, attn_ms, pre_ms = max_over_ranks([step_ms, attn_ms, pre_ms], pg, dev)

    # ---- end to end through the public API with pinned host buffers
    qh, kh, vh = (x.cpu().pin_memory() for x in (qd, kd, vd))
    oh = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    for _ in range(2):
        sageattn(qh, kh, vh, w.layout, w.is_causal, None, w.smooth_k, w.smooth_q, w.smooth_v, out=oh,
                 qk_bits=w.qk_bits)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(3, min(args.steps, 10))
    e0.record(stream)
    for _ in range(e2e_steps):
        sageattn(qh, kh, vh, w.layout, w.is_causal, None, w.smooth_k, w.smooth_q, w.smooth_v, out=oh,
                 qk_bits=w.qk_bits)
    e1.record(stream)
    barrier()
    e2e_ms, = max_over_ranks([e0.elapsed_time(e1) / e2e_steps], pg, dev)

    bf16_tflops, hbm_gbs, peak_src = _peaks()
    peak8 = 2.0 * bf16_tflops  # 8-bit dense = 2 x bf16 dense (nominal 4.5 / 2.25 PFLOP/s)
    achieved = w.ops / (attn_ms * 1e-3) / 1e12
    value = replica_value(world, w.ops, step_ms)
    mma_peak = mma_loop_peak(dev)
    kernels_per_step = 4 + (1 if w.smooth_q else 0)  # kv_stats, kv_finalize, quantize, (delta_s), attention

    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("i8xi8->i32 (QK)" if w.qk_bits == 8 else "i4 codes in i8xi8->i32 (QK)") + ", e4m3xe4m3->f32 (PV)",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "Nkv": w.Nkv,
                   "D": w.D, "layout": w.layout, "input_dtype": w.dtype, "causal": w.is_causal,
                   "smooth_k": w.smooth_k, "qk_bits": w.qk_bits, "parallelism": f"replicas x{world}",
                   "l2": f"inputs {in_bytes / 2**20:.0f} MiB > 126 MiB L2 (no flush)"},
        "roofline": {"bound": "tensor", "kernel": "attn_fwd_kernel", "achieved": achieved,
                     "peak": peak8, "unit": "TFLOP/s", "frac": achieved / peak8, "traffic": _attn_traffic(w),
                     "peak_source": f"{peak_src} bf16 x 2 (burst)",
                     "peak_measured_mma_loop": mma_peak,
                     "frac_of_mma_loop_i8": achieved / mma_peak["i8"],
                     "attn_ms": attn_ms, "prepass_ms": pre_ms,
                     "prepass_gbs": _prepass_bytes(w, qd, kd, vd) / (pre_ms * 1e-3) / 1e9},
        "e2e": {"value": replica_value(world, w.ops, e2e_ms), "unit": "TOPS",
                "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out.numel() * 2},
        "clocks": clocks,
        "gpu_launches": kernels_per_step * args.steps,
    }
    if rank == 0 and not args.no_cpu_baseline:
        heads, tiles = _sample_size(w, 12.0)
        tops, dt, desc, threads = oracle_sample(w, heads, tiles)
        line["cpu_baseline"] = {"value": tops, "unit": "TOPS", "cores": threads, "kind": "oracle",
                                "sample": desc + f" ({dt:.1f} s)"}
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# A variable-length batch (packed sequences): 16 sequences of H32 D128 bf16
# whose query and key lengths are drawn uniformly from [256, 4096] (seeded),
# non-causal, smooth_k.  No single configuration of the pages is variable
# length; this stands in for their "variable sequence lengths per batch".
VARLEN = dict(name="varlen_16seq_256to4096_h32_d128_bf16", nseq=16, H=32, D=128, dtype="bf16",
              lo=256, hi=4096, seed=4)


def run_varlen(args):
    """`--varlen`: the same JSON line for the variable-length batch above
    (one process, one GPU)."""
    import torch
    from quantized_attention_subtract_b200 import binding
    from quantized_attention_subtract_b200.workloads import generate_varlen
    c = VARLEN
    rng = np.random.default_rng(c["seed"])
    lq = rng.integers(c["lo"], c["hi"] + 1, c["nseq"])
    lk = rng.integers(c["lo"], c["hi"] + 1, c["nseq"])
    cu_q, cu_kv, q, k, v = generate_varlen(c["H"], c["H"], c["D"], lq, lk, c["dtype"], seed=c["seed"])
    ops = float(4.0 * c["H"] * c["D"] * np.sum(lq.astype(np.float64) * lk))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    to_dev = lambda x: torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    out = torch.empty_like(qd)
    p = binding.make_varlen_params(qd, kd, vd, out, cu_q, cu_kv)
    ws = binding.alloc_workspace(p, dev)
    stream = torch.cuda.current_stream(dev)
    clk = ClockSampler(0)
    clk.start()
    for _ in range(args.warmup):
        binding.attn_fwd(p, dev)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk.mark_begin()
    e0.record(stream)
    for _ in range(args.steps):
        binding.attn_fwd(p, dev)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clk.mark_end()
    step_ms = e0.elapsed_time(e1) / args.steps
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(args.steps)]
    for a_, b_, c_ in evs:
        a_.record(stream)
        binding.attn_fwd_prepass(p, dev)
        b_.record(stream)
        binding.attn_fwd_attention(p, dev)
        c_.record(stream)
    torch.cuda.synchronize(dev)
    pre_ms = float(np.mean([x.elapsed_time(y) for x, y, _ in evs]))
    attn_ms = float(np.mean([y.elapsed_time(z) for _, y, z in evs]))
    clk.stop()
    assert binding.device_status(p) == 0, "device status nonzero"
    # end to end: inputs from pinned host buffers and the output back, per step
    qh, kh, vh = (x.cpu().pin_memory() for x in (qd, kd, vd))
    oh = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    e2e_steps = max(3, min(args.steps, 10))
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(e2e_steps):
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        binding.attn_fwd(p, dev)
        oh.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    bf16_tflops, _, peak_src = _peaks()
    peak8 = 2.0 * bf16_tflops
    achieved = ops / (attn_ms * 1e-3) / 1e12
    in_bytes = 2 * (qd.numel() + kd.numel() + vd.numel())
    line = {
        "metric": METRIC, "value": ops / (step_ms * 1e-3) / 1e12, "unit": "TOPS", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8xi8->i32 (QK), e4m3xe4m3->f32 (PV)",
        "data": "synthetic",
        "config": {"workload": c["name"], "sequences": c["nseq"], "Hq": c["H"], "Hkv": c["H"],
                   "D": c["D"], "total_q": int(cu_q[-1]), "total_kv": int(cu_kv[-1]),
                   "max_q": int(lq.max()), "max_kv": int(lk.max()), "layout": "packed [total, H, D]",
                   "input_dtype": c["dtype"], "causal": False, "smooth_k": True,
                   "parallelism": "replicas x1",
                   "l2": f"inputs {in_bytes / 2**20:.0f} MiB > 126 MiB L2 (no flush)"},
        "roofline": {"bound": "tensor", "kernel": "attn_fwd_kernel", "achieved": achieved, "peak": peak8,
                     "unit": "TFLOP/s", "frac": achieved / peak8, "traffic": None,
                     "peak_source": f"{peak_src} bf16 x 2 (burst)", "attn_ms": attn_ms,
                     "prepass_ms": pre_ms},
        "e2e": {"value": ops / (e2e_ms * 1e-3) / 1e12, "unit": "TOPS", "h2d_bytes_per_step": in_bytes,
                "d2h_bytes_per_step": out.numel() * 2},
        "clocks": clk.summary(),
        "gpu_launches": 4 * args.steps,
    }
    if not args.no_cpu_baseline:
        # the oracle on a bounded sample of the first sequence (a batched
        # problem of its shape, inputs drawn the same way)
        w0 = Workload(c["name"] + "_seq0", 1, c["H"], c["H"], int(lq[0]), int(lk[0]), c["D"], "HND",
                      c["dtype"], k_offset_sigma=3.0, seed=c["seed"])
        heads, tiles = _sample_size(w0, 12.0)
        tops, dt, desc, threads = oracle_sample(w0, heads, tiles)
        line["cpu_baseline"] = {"value": tops, "unit": "TOPS", "cores": threads, "kind": "oracle",
                                "sample": desc + f" ({dt:.1f} s)"}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--varlen", action="store_true",
                    help="time the variable-length batch instead of --workload (one GPU)")
    ap.add_argument("--qk-bits", type=int, default=8, choices=[8, 4],
                    help="bits of the Q and K codes (4: the INT4 variant)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = WORKLOADS[args.workload].with_(qk_bits=args.qk_bits)
    if args.varlen and args.impl == "ours":
        run_varlen(args)
        return
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()

"""Benchmark: effective attention TFLOP/s (4 * d * ||M||_0 per (b, head)) of
the sliding-window prefill on the Mistral-style workload (B=2, Hq=32, Hkv=8,
N=8192, d=128, W=4096), plus the other workloads as `variants` (local +
strided prefill, differential prefill, long-context SWA prefill, and the
decode step's HBM GB/s).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One process per GPU (torchrun for N > 1, NCCL only for the barrier and the
max-over-ranks time). The path shards over batches: every rank runs the same
per-GPU workload on its own seeded inputs, with no data exchange (weak
scaling). Timing: CUDA events on the launching stream around each step; an
L2 flush (a 512 MiB write) runs between steps outside the events.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "effective attention TFLOPS (4*d*nnz(M)), SWA prefill"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
_CSRC = "differential_attention_swa_b200/csrc/"
PREFILL_SOURCES = [_CSRC + f for f in ("prefill.cu", "ptx.cuh", "schedule.cuh", "internal.h")]
DECODE_SOURCES = [_CSRC + f for f in ("decode.cu", "ptx.cuh", "internal.h")]
DIFF_DECODE_SOURCES = [_CSRC + f for f in ("diff_decode.cu", "ptx.cuh", "internal.h")]
BWD_SOURCES = [_CSRC + f for f in ("backward.cu", "ptx.cuh", "schedule.cuh", "internal.h")]
# the committed ncu summary of each workload's dominant kernel (profiles/):
# its DRAM bytes per launch count as `roofline.traffic` while the kernel's
# sources still hash to the value the summary records
PROFILES = {
    "mistral_swa_prefill": ("prefill_swa_mistral.md", PREFILL_SOURCES),
    "gemma_swa_prefill": ("prefill_swa_gemma.md", PREFILL_SOURCES),
    "diff_causal": ("prefill_diff_causal.md", PREFILL_SOURCES),
    "local_strided_prefill": ("prefill_strided_local.md", PREFILL_SOURCES),
    "longformer_global_prefill": ("prefill_global_longformer.md", PREFILL_SOURCES),
    "longformer_dilated_prefill": ("prefill_dilated_longformer.md", PREFILL_SOURCES),
    "mistral_swa_backward": ("backward_swa_mistral.md", BWD_SOURCES),
    "local_strided_backward": ("backward_strided_local.md", BWD_SOURCES),
    "gemma_swa_decode": ("decode_gemma.md", DECODE_SOURCES),
    "diff_gqa_decode": ("decode_diff_gqa.md", DIFF_DECODE_SOURCES),
}


def workload_traffic(name: str) -> float | None:
    if name not in PROFILES:
        return None
    return profiled_traffic(*PROFILES[name])


# ------------------------------------------------------------ host logic --

def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only", default=None, help="run one workload by name (profiling)")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"]))}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def source_hash(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(summary: str, sources) -> float | None:
    """DRAM bytes per launch from a committed ncu summary, if the kernel's
    sources still hash to what the summary records (else None)."""
    path = os.path.join(ROOT, "profiles", summary)
    try:
        text = open(path).read()
    except OSError:
        return None
    m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    s = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
    if not m or not s or s.group(1) != source_hash(sources):
        return None
    return float(m.group(1))


def aggregate(per_rank_ms, units_per_rank):
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    n = len(per_rank_ms)
    t = max(per_rank_ms)
    return n * units_per_rank / (t * 1e-3), t


def max_over_ranks(ms: float, dist, device="cpu") -> float:
    """The slowest rank's time (every rank takes part in the same all-reduce)."""
    if dist is None:
        return ms
    import torch

    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_seed(base: int, rank: int) -> int:
    """Each rank draws its own batch (weak scaling over data)."""
    return base + 1000 * rank


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = bus_id
        self.proc = None
        self.lines = []

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "20"]
        if self.bus_id:
            cmd[1:1] = ["-i", self.bus_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        return self.summary()

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[3], parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        loaded = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[4]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "power_w_max": max(r[2] for r in rows)}


# ---------------------------------------------------------- measurement --

def flush_l2(buf):
    buf.add_(1)


def time_steps(fn, steps, warmup, flush_buf, stream):
    import torch

    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        flush_l2(flush_buf)
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def prefill_workload(name, rank):
    import torch

    import differential_attention_swa_b200 as swa
    from differential_attention_swa_b200.inputs import WORKLOADS, attn_inputs, diff_inputs

    w = WORKLOADS[name]
    seed = shard_seed(0, rank)
    if w.kind == "diff":
        ins = [t.cuda() for t in diff_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.dv, seed=seed)]
        lam = torch.full((w.Hq,), w.lam, dtype=torch.float32, device="cuda")
        out = torch.empty((w.B, w.Hq, w.N, w.dv_), dtype=torch.bfloat16, device="cuda")
        call = lambda xs, o: swa.diff_attn_fwd(*xs, lam, window=w.W, scale=w.scale, out=o)
        nnz = swa.count_nonmasked(swa.MASK_WINDOW, w.N, w.W)
        flops = nnz * w.B * w.Hq * 2 * (2 * w.d + 2 * w.dv_)  # two maps, each 2*d_qk + 2*d_v per cell
    elif w.kind == "swa_bwd":
        from differential_attention_swa_b200.inputs import randn_bf16

        q, k, v = (t.cuda() for t in attn_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=seed))
        d_o = randn_bf16((w.B, w.Hq, w.N, w.d), seed + 3).cuda()
        # the forward, outside the timed region (S > 0: the local + strided mask)
        if w.S:
            o, lse = swa.strided_attn_fwd(q, k, v, w.W, w.S, return_lse=True)
            ws_bytes = int(swa.library().strided_attn_bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d, w.S))
            nnz = swa.count_nonmasked(swa.MASK_STRIDED, w.N, w.W, w.S)
        else:
            o, lse = swa.swa_attn_fwd(q, k, v, w.W, return_lse=True)
            ws_bytes = swa.attn_bwd_workspace_bytes(w.B, w.Hq, w.N)
            nnz = swa.count_nonmasked(swa.MASK_WINDOW, w.N, w.W)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        out = None
        call = lambda xs, _o: swa.swa_attn_bwd(*xs[:6], w.W, workspace=xs[6], stride=w.S)
        # the usual accounting: scores, dP, dV, dQ, dK = 5 products of 2*d per cell
        flops = 10 * w.d * nnz * w.B * w.Hq
        ins = [q, k, v, o, d_o, lse, ws]
    else:
        q, k, v = (t.cuda() for t in attn_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=seed))
        out = torch.empty_like(q)
        if w.kind == "swa":
            call = lambda xs, o: swa.swa_attn_fwd(*xs, w.W, out=o)
            nnz = swa.count_nonmasked(swa.MASK_WINDOW, w.N, w.W)
        elif w.kind == "global":  # S carries the number of global tokens
            call = lambda xs, o: swa.global_attn_fwd(*xs, w.W, w.S, out=o)
            nnz = swa.count_nonmasked(swa.MASK_GLOBAL, w.N, w.W, w.S)
        elif w.kind == "dilated":  # S carries the dilation; each row sees min(W, i // S + 1) keys
            call = lambda xs, o: swa.dilated_attn_fwd(*xs, w.W, w.S, out=o)
            nnz = sum(min(w.W, i // w.S + 1) for i in range(w.N))
        else:
            call = lambda xs, o: swa.strided_attn_fwd(*xs, w.W, w.S, out=o)
            nnz = swa.count_nonmasked(swa.MASK_STRIDED, w.N, w.W, w.S)
        flops = 4 * w.d * nnz * w.B * w.Hq
        ins = [q, k, v]
    fn = lambda: call(ins, out)
    return w, fn, call, flops, ins, out


def decode_workload(rank, name="gemma_swa_decode"):
    import torch

    import differential_attention_swa_b200 as swa
    from differential_attention_swa_b200.inputs import WORKLOADS, decode_inputs

    w = WORKLOADS[name]
    if w.kind == "diff_decode":
        return diff_decode_workload(rank, w)
    n_sink = int(w.extra.get("n_sink", 0))
    T = w.steps
    q, kn, vn, kc, vc = decode_inputs(T, w.B, w.Hq, w.Hkv, w.d, n_sink + w.W, seed=shard_seed(0, rank))
    q, kn, vn, kc, vc = (t.cuda() for t in (q, kn, vn, kc, vc))
    pos = torch.tensor([[w.pos0 + t] * w.B for t in range(T)], dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    ws = torch.empty(max(16, swa.sink_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.d, n_sink, w.W)),
                     dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()

    def steps():
        for t in range(T):
            if n_sink:
                swa.swa_sink_decode_step(q[t], kn[t], vn[t], kc, vc, pos[t], n_sink, out=out[t], workspace=ws,
                                         scale=w.scale)
            else:
                swa.swa_decode_step(q[t], kn[t], vn[t], kc, vc, pos[t], out=out[t], workspace=ws, scale=w.scale)

    with torch.cuda.stream(stream):
        steps()  # warm (also sets kernel attributes before capture)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        steps()
    # bytes per step: K and V of every cached slot read once per KV head, the
    # query and output rows, the new token's K and V
    kv = 2 * w.B * w.Hkv * (n_sink + w.W) * w.d * 2
    qo = 2 * w.B * w.Hq * w.d * 2
    new = 2 * w.B * w.Hkv * w.d * 2
    bytes_per_step = kv + qo + new
    return w, g, bytes_per_step, T


def diff_decode_workload(rank, w):
    import torch

    import differential_attention_swa_b200 as swa
    from differential_attention_swa_b200.inputs import diff_decode_inputs

    T, dk, dv = w.steps, w.d, w.dv_
    ins = diff_decode_inputs(T, w.B, w.Hq, w.Hkv, dk, dv, w.W, seed=shard_seed(0, rank))
    q1, q2, k1n, k2n, vn, k1c, k2c, vc = (t.cuda() for t in ins)
    lam = torch.full((w.Hq,), w.lam, dtype=torch.float32, device="cuda")
    pos = torch.tensor([[w.pos0 + t] * w.B for t in range(T)], dtype=torch.int32, device="cuda")
    out = torch.empty((T, w.B, w.Hq, dv), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(16, swa.diff_decode_workspace_bytes(w.B, w.Hq, w.Hkv, dk, dv, w.W)), dtype=torch.uint8,
                     device="cuda")
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()

    def steps():
        for t in range(T):
            swa.swa_diff_decode_step(q1[t], q2[t], k1n[t], k2n[t], vn[t], k1c, k2c, vc, pos[t], lam, out=out[t],
                                     workspace=ws, scale=w.scale)

    with torch.cuda.stream(stream):
        steps()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        steps()
    # bytes per step: K1, K2 and V of every cached slot read once per KV head
    # (V once for both maps), both maps' query rows, the output row, the new
    # token's K1, K2 and V, and lambda
    kv = w.B * w.Hkv * w.W * (2 * dk + dv) * 2
    qo = w.B * w.Hq * (2 * dk + dv) * 2
    new = w.B * w.Hkv * (2 * dk + dv) * 2
    return w, g, kv + qo + new + 4 * w.Hq, T


def prefill_kernel_name(w) -> str:
    """The prefill kernel instantiation a workload runs (for the roofline label)."""
    if w.kind == "swa_bwd":
        return f"bwd_dkdv_kernel<{w.d}> + bwd_dq_kernel<{w.d}>"
    if w.kind == "diff":
        return f"prefill_kernel<{w.d},{w.dv_},diff>"
    gen = ",global" if w.kind == "global" else (",row views" if w.kind == "dilated" else "")
    pairs = ",kv pairs" if (w.Hq // w.Hkv) % 2 == 1 and w.Hq % 2 == 0 and w.d == 64 else ""
    return f"prefill_kernel<{w.d},{w.d}{gen}{pairs}>"


def launches_per_step(w) -> int:
    """Kernels one step of a workload launches: the persistent prefill kernel,
    or the backward's row-statistics pass, the stride keys' dK/dV pass (local
    + strided mask only), the dK/dV kernel and the dQ kernel."""
    if w.kind == "swa_bwd":
        return 3 + (1 if w.S else 0)
    return 1


def measure_ours(args, rank, world, peaks, peak_src, dist):
    import torch

    import differential_attention_swa_b200 as swa

    swa.library()
    stream = torch.cuda.current_stream()
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    bus = None
    if hasattr(props, "pci_bus_id"):
        bus = f"{getattr(props, 'pci_domain_id', 0):08X}:{props.pci_bus_id:02X}:{getattr(props, 'pci_device_id', 0):02X}.0"

    main_name = args.only or "mistral_swa_prefill"
    if main_name.endswith("_decode"):
        return measure_decode_only(args, rank, world, peaks, flush, stream, main_name)
    w, fn, call, flops, ins, out = prefill_workload(main_name, rank)
    clocks = ClockSampler(bus)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    ms = time_steps(fn, args.steps, max(3, args.warmup), flush, stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if dist:
        dist.barrier()
    err = swa.last_device_error()
    if err != swa.OK:
        raise RuntimeError(f"kernel reported status {err}")
    mean_ms = sum(ms) / len(ms)
    t_all = [max_over_ranks(mean_ms, dist, "cuda")] * world
    value, tmax = aggregate(t_all, flops)
    achieved = flops / (mean_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    traffic = workload_traffic(main_name)
    res = {
        "metric": METRIC if main_name == "mistral_swa_prefill" else f"effective attention TFLOPS, {main_name}",
        "value": round(value / 1e12, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(tmax, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic N(0,1) bf16, seeded per rank",
        "config": {"workload": main_name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "W": w.W,
                   "S": w.S, "parallelism": f"dp{world} (independent batches)", "l2": "flushed between steps"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_source": f"{peak_src} bf16 burst (MEASURED_PEAKS.json)" if peak_src == "measured"
                     else "fallback 1.59 PFLOP/s",
                     "kernel": prefill_kernel_name(w)},
        "clocks": clk,
        "gpu_launches": args.steps * launches_per_step(w),
    }
    if not args.no_e2e and out is not None:  # the backward workload has no single output to copy back
        res["e2e"] = whole_job_e2e(measure_e2e(call, ins, out, flops, stream), flops, world, dist, "cuda")
    if not args.no_variants and args.only is None:
        res["variants"] = measure_variants(args, rank, peaks, flush, stream)
    return res


def whole_job_e2e(e2e, flops, world, dist, device="cpu"):
    """A rank's end-to-end record turned whole-job: the slowest rank's step
    time, every rank's work and copied bytes (weak scaling). Every rank calls
    it, so every rank takes part in the one collective."""
    t = max_over_ranks(e2e["ms_raw"], dist, device)
    value, tmax = aggregate([t] * world, flops)
    out = dict(e2e)
    out.pop("ms_raw")
    out["value"] = round(value / 1e12, 3)
    out["ms_per_step"] = round(tmax, 4)
    out["h2d_bytes_per_step"] = e2e["h2d_bytes_per_step"] * world
    out["d2h_bytes_per_step"] = e2e["d2h_bytes_per_step"] * world
    return out


def measure_e2e(call, ins, out, flops, stream, steps=8):
    """Same metric through the public call with host buffers: every step
    copies its inputs in from pinned host memory, runs the call and copies
    its output back. Steps are pipelined over two sets of device buffers on
    three streams (inputs of step k+1 go in while step k computes and step
    k-1's output comes back), as a serving loop would; the timed region runs
    from the first input copy to the last output copy."""
    import torch

    hosts = [t.cpu().pin_memory() for t in ins]
    host_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    dev_in = [list(ins), [torch.empty_like(t) for t in ins]]
    dev_out = [out, torch.empty_like(out)]
    h2d = sum(t.numel() * t.element_size() for t in hosts)
    d2h = out.numel() * out.element_size()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for k in range(n):
            b = k % 2
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(ev_comp[b])  # step k-2 has finished reading these inputs
                for h, d in zip(hosts, dev_in[b]):
                    d.copy_(h, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if k >= 2:
                stream.wait_event(ev_out[b])  # step k-2's output has been copied out
            call(dev_in[b], dev_out[b])
            ev_comp[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                host_out[b].copy_(dev_out[b], non_blocking=True)
                ev_out[b].record(s_out)

    run(2)
    torch.cuda.synchronize()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    run(steps)
    z.record(s_out)
    torch.cuda.synchronize()
    ms = a.elapsed_time(z) / steps
    return {"value": round(flops / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
            "ms_raw": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelined": "2 buffer sets, 3 streams"}


def measure_decode_only(args, rank, world, peaks, flush, stream, name):
    v = measure_decode(args, rank, peaks, flush, stream, name=name)
    return {"metric": "decode HBM GB/s", "value": v["value"], "unit": "GB/s", "n_gpus": world, "steps": v["steps"],
            "ms_per_step": v["ms_per_step"], "roofline": v["roofline"], "config": {"workload": name}}


def measure_decode(args, rank, peaks, flush, stream, reps=5, name="gemma_swa_decode"):
    import torch

    w, g, bytes_per_step, T = decode_workload(rank, name)
    diff = w.kind == "diff_decode"
    ms = time_steps(lambda: g.replay(), reps, 3, flush, stream)
    mean_ms = sum(ms) / len(ms)
    gbs = bytes_per_step * T / (mean_ms * 1e-3) / 1e9
    peak = peaks["hbm_gbs"]
    del g
    torch.cuda.synchronize()
    return {"value": round(gbs, 1), "unit": "GB/s", "ms_per_step": round(mean_ms / T, 5), "steps": reps,
            "decode_steps_per_graph": T, "bytes_per_decode_step": bytes_per_step,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(gbs / peak, 4),
                         "traffic": workload_traffic(name),
                         "kernel": ("diff_decode_split_kernel<2> + diff_decode_combine_kernel" if diff else
                                    "decode_split_kernel<128,2> + decode_combine_kernel<128>")},
            "launches": reps * T * 2}


def measure_variants(args, rank, peaks, flush, stream):
    import torch

    import differential_attention_swa_b200 as swa

    out = {}
    reps = max(5, min(args.steps, 10))
    for name in ("local_strided_prefill", "diff_causal", "gemma_swa_prefill", "longformer_global_prefill",
                 "longformer_dilated_prefill", "mistral_swa_backward", "local_strided_backward"):
        w, fn, _call, flops, ins, o = prefill_workload(name, rank)
        ms = time_steps(fn, reps, 3, flush, stream)
        mean_ms = sum(ms) / len(ms)
        tf = flops / (mean_ms * 1e-3) / 1e12
        traffic = workload_traffic(name)
        out[name] = {"value": round(tf, 3), "unit": "TFLOP/s", "ms_per_step": round(mean_ms, 4), "steps": reps,
                     "algorithmic_flops": flops,
                     "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": peaks["bf16_tflops"],
                                  "unit": "TFLOP/s", "frac": round(tf / peaks["bf16_tflops"], 4),
                                  "traffic": traffic, "kernel": prefill_kernel_name(w)},
                     "launches": reps}
        del ins, o, fn
        torch.cuda.empty_cache()
    out["gemma_swa_decode"] = measure_decode(args, rank, peaks, flush, stream)
    out["gemma_sink_decode"] = measure_decode(args, rank, peaks, flush, stream, name="gemma_sink_decode")
    out["diff_gqa_decode"] = measure_decode(args, rank, peaks, flush, stream, name="diff_gqa_decode")
    if swa.last_device_error() != swa.OK:
        raise RuntimeError("a variant kernel reported an error")
    return out


# ------------------------------------------------------------- the oracle --

def oracle_sample(w, rows_n, seed, inputs=None):
    """Times the fp64 oracle on `rows_n` seeded rows of the workload; returns
    (seconds, attended cells, flops) for those rows."""
    import numpy as np

    import oracle
    from differential_attention_swa_b200.inputs import attn_inputs

    if inputs is None:
        inputs = attn_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=0)
    q, k, v = inputs
    rng = np.random.default_rng(seed)
    rows = rng.integers(0, w.B * w.Hq * w.N, rows_n)
    i = rows % w.N
    cells = int(np.minimum(i + 1, w.W).sum())
    t0 = time.perf_counter()
    oracle.attention(w.kind, q, k, v, W=w.W, S=w.S, scale=w.scale, rows=rows)
    dt = time.perf_counter() - t0
    return dt, cells, 4 * w.d * cells


def cpu_baseline(min_seconds=10.0):
    import oracle
    from differential_attention_swa_b200.inputs import WORKLOADS, attn_inputs

    w = WORKLOADS["mistral_swa_prefill"]
    inputs = attn_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=0)
    n = 512
    while True:
        dt, cells, flops = oracle_sample(w, n, 123, inputs)
        if dt >= min_seconds or n >= 1 << 19:
            break
        n = int(n * max(2.0, 1.2 * min_seconds / max(dt, 1e-3)))
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.default_threads(),
            "kind": "oracle",
            "sample": f"{n} seeded rows (of {w.B * w.Hq * w.N}) of mistral_swa_prefill, fp64, {dt:.1f} s"}


def run_reference(args):
    """The reference arm: the fp64 oracle as it stands on the host cores."""
    import oracle

    world = int(os.environ.get("WORLD_SIZE", "1"))
    from differential_attention_swa_b200.inputs import WORKLOADS, attn_inputs

    w = WORKLOADS["mistral_swa_prefill"]
    inputs = attn_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=0)
    rows_per_step = 256
    for s in range(max(3, args.warmup)):
        oracle_sample(w, rows_per_step, 10_000 + s, inputs)
    times, flops = [], 0
    for s in range(args.steps):
        dt, _, f = oracle_sample(w, rows_per_step, s, inputs)
        times.append(dt)
        flops += f
    total = sum(times)
    value = flops / total / 1e12
    sample = f"{rows_per_step} seeded rows of mistral_swa_prefill per step, fp64"
    return {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": round(1e3 * total / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic N(0,1) bf16 widened to fp64",
            # the config of this arm's comparison line: the same as the GPU
            # arm's for the same launch (what the oracle actually ran is in
            # cpu_baseline.sample)
            "config": {"workload": "mistral_swa_prefill", "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                       "W": w.W, "S": w.S, "parallelism": f"dp{world} (independent batches)",
                       "l2": "flushed between steps"},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.default_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ main --

def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    import torch

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist

        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    peaks, peak_src = load_peaks()
    res = measure_ours(args, rank, world, peaks, peak_src, dist)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.only is None:
        res["cpu_baseline"] = cpu_baseline()
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())

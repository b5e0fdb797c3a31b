"""Benchmark of the fused attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One step = one pass of the whole hot path over one batch of the LLaMA-7B
attention-layer workload (B=2, Hq=Hkv=32, N=2048, D=128, fp16,
scale=1/sqrt(128)): the non-causal forward pass and the causal forward pass,
both through the library's C ABI.  Inputs are synthetic (seeded N(0,1),
rounded to fp16) and resident in HBM when timing starts; L2 is flushed
(256 MiB write, outside the timed events) before every pass because the
inputs (~100 MB) fit in L2.  Beside the step, every other workload of the
pages is timed on its own (the tiny check, the sequence sweep, the GQA/MQA and
head-dim sweep, the 128K context) together with KV-cache decode, key windows,
a score bias and the backward pass.

metric: attention forward TFLOP/s with FLOPs = 4*B*Hq*Nq*Nk*D (halved for the
causal pass).  Prints one JSON line on rank 0.  For N > 1 (torchrun) every rank
runs an independent copy of the workload (weak scaling, no data-path
collective); time is the max over ranks.

--impl reference times the CPU oracle (plain three-pass fp64 attention) on the
host cores on bounded row samples of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attn fwd TFLOP/s (4·B·Hq·Nq·Nk·D, ½ if causal) and % of B200 dense FP16 peak"
SPEC_PEAK_TFLOPS = 2250.0
FALLBACK_PEAK_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload lines (tiny, sweep, GQA/head-dim, 128K)")
    ap.add_argument("--no-decode", action="store_true", help="skip the KV-cache decode measurement")
    ap.add_argument("--no-window", action="store_true",
                    help="skip the sliding-window measurement")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward-pass measurement")
    ap.add_argument("--no-bias", action="store_true", help="skip the score-bias measurement")
    ap.add_argument("--no-unfused", action="store_true",
                    help="skip the unfused (standard attention) comparison")
    return ap.parse_args()


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank measurement over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flops_per_step: float, steps: int, max_ms: float, world: int) -> float:
    """Whole-job throughput: every rank runs its own replica of the workload."""
    return world * flops_per_step * steps / (max_ms * 1e-3) / 1e12


def workloads():
    from fa_inputs import llama7b
    return [llama7b(False), llama7b(True)]


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"])
    return FALLBACK_HBM_GBS


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    return FALLBACK_PEAK_TFLOPS, 1400.0, "fallback"


# The sources the forward kernel is built from (the traffic record is about it).
FWD_KERNEL_SOURCES = ("fa_fwd_sm100.cu", "sm100_ptx.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "tiled_attention_15_b200", "csrc")
    for n in FWD_KERNEL_SOURCES:
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it matches the current kernel."""
    p = os.path.join(ROOT, "profiles", "fa_fwd_d128_llama7b_traffic.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    with open(p) as f:
        for line in f:
            if "=" in line and not line.startswith("#"):
                a, b = line.split("=", 1)
                kv[a.strip()] = b.strip()
    if kv.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """NVML samples of SM clock and clock-event reasons while the GPU works.

    Runs from the warm-up to the end of the per-workload lines; summary() gives
    the median SM clock and the union of throttle reasons over all samples, and
    how many of them fell inside the timed region of the step (an NVML query
    takes a few ms, so a short timed region gets only a few)."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int):
        self.ok = False
        self.samples = []  # (time, mhz, reason bits)
        self.window = [None, None]
        self.sections = []
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, r))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.001)

    def mark(self, i: int):
        """Mark the start (0) or end (1) of the timed region."""
        self.window[i] = time.perf_counter()

    def section(self, name: str):
        """Start a named section (it ends where the next one starts)."""
        self.sections.append((name, time.perf_counter()))

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        busy = [x for x in self.samples if not x[2] & 0x1]  # gpu_idle samples left out
        if not self.ok or not busy:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        reasons = set()
        for _, _, r in busy:
            reasons |= {n for b, n in self.REASONS.items() if r & b}
        t0, t1 = self.window
        timed = [m for t, m, _ in busy if t0 is not None and t1 is not None and t0 <= t <= t1]
        per_section = {}
        bounds = self.sections + [("", float("inf"))]
        for (name, a), (_, b) in zip(bounds[:-1], bounds[1:]):
            xs = [m for t, m, _ in busy if a <= t < b]
            if xs:
                per_section[name] = statistics.median(xs)
        return {"sm_mhz": statistics.median(m for _, m, _ in busy), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(busy),
                "timed_region_samples": len(timed),
                "timed_region_sm_mhz": statistics.median(timed) if timed else None,
                "sm_mhz_by_section": per_section,
                "window": "warm-up through the per-workload lines (GPU busy)"}


# ----------------------------------------------------------------------------- reference arm
def oracle_sample(ws, rows_per_head: int, seed: int, qkv=None):
    """Run the oracle on a seeded sample of query rows of every head; returns (flops, seconds)."""
    import numpy as np
    import oracle
    from fa_inputs import make_qkv, sample_rows
    flops, secs = 0.0, 0.0
    for w in ws:
        q, k, v = qkv if qkv is not None else make_qkv(w)
        rows = sample_rows(w.Nq, rows_per_head, seed)
        vis = np.minimum(rows + 1, w.Nk) if w.causal else np.full(len(rows), w.Nk)
        flops += 4.0 * w.D * float(vis.sum()) * w.B * w.Hq
        t0 = time.perf_counter()
        oracle.attention(q, k, v, w.softmax_scale, w.causal, rows=rows)
        secs += time.perf_counter() - t0
    return flops, secs


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import oracle
    from fa_inputs import make_qkv
    ws = workloads()
    qkv = make_qkv(ws[0])  # both passes use the same seed-0 draws
    rows = 32
    for i in range(args.warmup):
        oracle_sample(ws, rows, 1000 + i, qkv)
    flops = secs = 0.0
    for i in range(args.steps):
        f, s = oracle_sample(ws, rows, i, qkv)
        flops += f
        secs += s
    tflops = flops / secs / 1e12
    cores = oracle.max_threads()
    sample = (f"{rows} seeded query rows per (b, head) of each pass (non-causal, causal) per step; "
              f"{args.steps} steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": tflops, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1), rounded to fp16)",
        "config": {"workload": "llama7b-attn B2 Hq32 Hkv32 N2048 D128 fp16, non-causal + causal",
                   "B": 2, "Hq": 32, "Hkv": 32, "N": 2048, "D": 128},
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- CUDA arm
def device_qkv(w, dev, seed):
    """Seeded N(0,1) inputs drawn on the device (the large sweep workloads; same recipe
    as fa_inputs.make_qkv, including the outlier keys, but torch's generator)."""
    import torch
    g = torch.Generator(device=dev).manual_seed(seed)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
    q = torch.randn((w.B, w.Hq, w.Nq, w.D), device=dev, generator=g) * w.q_mult
    k = torch.randn((w.B, w.Hkv, w.Nk, w.D), device=dev, generator=g)
    v = torch.randn((w.B, w.Hkv, w.Nk, w.D), device=dev, generator=g)
    if w.outlier_frac > 0.0:
        n_out = int(w.outlier_frac * w.Nk)
        for b in range(w.B):
            for h in range(w.Hkv):
                rows = torch.randperm(w.Nk, device=dev, generator=g)[:n_out]
                k[b, h, rows] *= w.outlier_mult
    return q.to(dt), k.to(dt), v.to(dt)


def time_launches(fn, flush, stream, n=10, warm=3):
    """Median CUDA-event time (ms) of fn() over n launches, L2 flushed before each.

    All n launches are enqueued before the host waits, so the host-side cost of
    a call overlaps the GPU's previous work instead of opening a gap between an
    event and the kernel it brackets."""
    import torch
    for _ in range(warm):
        flush.zero_()
        fn()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        fn()
        b.record(stream)
    evs[-1][1].synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in evs)


def workload_line(w, ms, peak, hbm, flops=None):
    flops = w.flops() if flops is None else flops
    tf = flops / (ms * 1e-3) / 1e12
    gbs = w.io_bytes() / (ms * 1e-3) / 1e9
    return {"ms": round(ms, 4), "tflops": round(tf, 1), "frac_of_peak": round(tf / peak, 3),
            "alg_bytes": w.io_bytes(), "alg_gbs": round(gbs, 1), "frac_of_hbm": round(gbs / hbm, 3)}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    import tiled_attention_15_b200 as fa
    from fa_inputs import make_qkv

    assert args.warmup >= 3, "at least 3 warm-up steps"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        # a short timeout: a rank that fails makes the others' next collective
        # end with an error instead of waiting for good
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))

    def barrier():
        if world > 1:
            dist.barrier()

    peak, peak_sus, peak_kind = peaks()
    hbm = hbm_peak()
    ws = workloads()
    inputs = []
    for w in ws:
        q, k, v = make_qkv(w)
        inputs.append((w, q, k, v))
    # the non-causal and causal passes share the same Q, K, V draws (seed 0)
    q, k, v = (x.to(dev) for x in inputs[0][1:])
    outs = [(torch.empty_like(q), torch.empty(q.shape[:3], dtype=torch.float32, device=dev))
            for _ in ws]
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream

    def run_pass(j, qq=None, kk=None, vv=None, st=None):
        w, (o, lse) = ws[j], outs[j]
        fa.fa_fwd(q if qq is None else qq, k if kk is None else kk, v if vv is None else vv,
                  o=o, lse=lse, scale=w.softmax_scale, causal=w.causal,
                  stream=sptr if st is None else st)

    clk = ClockSampler(local)
    clk.__enter__()
    for _ in range(args.warmup):
        for j in range(len(ws)):
            flush.zero_()
            run_pass(j)
    torch.cuda.synchronize()
    assert fa.device_status(reset=True) == 0

    # ---- the timed step: each pass bracketed by its own events, L2 flushed before it
    K = args.steps
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in ws] for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    clk.section("step")
    clk.mark(0)
    for i in range(K):
        for j in range(len(ws)):
            flush.zero_()
            ev[i][j][0].record(stream)
            run_pass(j)
            ev[i][j][1].record(stream)
    torch.cuda.synchronize()
    clk.mark(1)
    barrier()
    per_pass = [[ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(K)] for j in range(len(ws))]
    total_ms = max_over_ranks(sum(sum(x) for x in per_pass), world, dev)
    assert fa.device_status(reset=True) == 0
    flops_step = sum(w.flops() for w in ws)
    value = aggregate_tflops(flops_step, K, total_ms, world)
    pass_lines = {("causal" if w.causal else "non-causal"):
                  {"median_ms": round(statistics.median(per_pass[j]), 5),
                   "tflops": round(w.flops() / (statistics.median(per_pass[j]) * 1e-3) / 1e12, 1),
                   "l2": "flushed before the pass"}
                  for j, w in enumerate(ws)}

    clk.section("e2e")
    # ---- end to end through the public API: pinned host inputs -> device -> both
    # passes -> O and LSE back to pinned host memory, every step.  Copies in and
    # out run on their own streams with two device buffer sets, so the upload of
    # step i + 1 and the download of step i - 1 overlap the passes of step i.
    hq, hk, hv = (x.pin_memory() for x in inputs[0][1:])
    ho = [[(torch.empty(q.shape, dtype=q.dtype, pin_memory=True),
            torch.empty(q.shape[:3], dtype=torch.float32, pin_memory=True)) for _ in ws]
          for _ in range(2)]
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    d2h = sum(a.numel() * a.element_size() + b.numel() * b.element_size() for a, b in ho[0])
    dbuf = [tuple(torch.empty_like(x) for x in (q, k, v)) for _ in range(2)]
    dout = [[(torch.empty_like(q), torch.empty(q.shape[:3], dtype=torch.float32, device=dev))
             for _ in ws] for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    E = max(10, K // 20)

    def e2e_run(n):
        done_in = [None, None]   # compute of the step that last read buffer b is done
        done_out = [None, None]  # download of the step that last wrote output set b is done
        for i in range(n):
            b = i & 1
            if done_in[b] is not None:
                s_in.wait_event(done_in[b])
            with torch.cuda.stream(s_in):
                for dst, src in zip(dbuf[b], (hq, hk, hv)):
                    dst.copy_(src, non_blocking=True)
            up = torch.cuda.Event()
            up.record(s_in)
            stream.wait_event(up)
            if done_out[b] is not None:
                stream.wait_event(done_out[b])
            for j, w in enumerate(ws):
                o, lse = dout[b][j]
                fa.fa_fwd(*dbuf[b], o=o, lse=lse, scale=w.softmax_scale, causal=w.causal,
                          stream=sptr)
            comp = torch.cuda.Event()
            comp.record(stream)
            done_in[b] = comp
            s_out.wait_event(comp)
            with torch.cuda.stream(s_out):
                for (o, lse), (h_o, h_l) in zip(dout[b], ho[b]):
                    h_o.copy_(o, non_blocking=True)
                    h_l.copy_(lse, non_blocking=True)
            down = torch.cuda.Event()
            down.record(s_out)
            done_out[b] = down
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    e2e_run(3)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_stream(stream)
    e2e_run(E)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = aggregate_tflops(flops_step, E, e2e_ms, world)
    assert fa.device_status(reset=True) == 0
    del dbuf, dout

    clk.section("backward")
    # ---- backward pass on the bench workload (LLaMA-7B layer), both passes
    backward = {}
    if not args.no_backward:
        g0 = torch.Generator(device=dev).manual_seed(1)
        bdo = torch.randn(q.shape, device=dev, dtype=q.dtype, generator=g0)
        bws = torch.empty(fa.load_library().fa_bwd_workspace_size(*q.shape[:3]), dtype=torch.uint8,
                          device=dev)
        bdq, bdk, bdv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        for w in ws:
            bo, bl = fa.fa_fwd(q, k, v, scale=w.softmax_scale, causal=w.causal, stream=sptr)
            ms = time_launches(lambda: fa.fa_bwd(q, k, v, bo, bl, bdo, scale=w.softmax_scale,
                                                 causal=w.causal, dq=bdq, dk=bdk, dv=bdv,
                                                 stream=sptr, workspace=bws), flush, stream)
            bflops = 2.5 * w.flops()  # five GEMMs against the forward pass's two
            backward["causal" if w.causal else "noncausal"] = {
                "ms": round(ms, 4), "tflops": round(bflops / (ms * 1e-3) / 1e12, 1),
                "frac_of_peak": round(bflops / (ms * 1e-3) / 1e12 / peak, 3)}
        # the same non-causal pass with one [N, N] score bias shared by all heads
        w = ws[0]
        g1 = torch.Generator(device=dev).manual_seed(2)
        bb = torch.randn((1, 1, w.Nq, w.Nk), device=dev, dtype=q.dtype, generator=g1)
        bo, bl = fa.fa_fwd(q, k, v, scale=w.softmax_scale, bias=bb, stream=sptr)
        ms = time_launches(lambda: fa.fa_bwd(q, k, v, bo, bl, bdo, scale=w.softmax_scale, dq=bdq,
                                             dk=bdk, dv=bdv, stream=sptr, workspace=bws, bias=bb),
                           flush, stream)
        bflops = 2.5 * w.flops()
        backward["noncausal_shared_bias"] = {
            "ms": round(ms, 4), "tflops": round(bflops / (ms * 1e-3) / 1e12, 1),
            "frac_of_peak": round(bflops / (ms * 1e-3) / 1e12 / peak, 3)}
        del bdo, bws, bdq, bdk, bdv, bb
        # head_dim 256: the GQA configuration's D = 256 variant (B4 Hq32 Hkv8 N8192 bf16 causal)
        from fa_inputs import gqa
        w = gqa(8, 256)
        gq, gk, gv = (x.to(dev) for x in make_qkv(w))
        gdo = torch.randn(gq.shape, device=dev, dtype=gq.dtype, generator=g0)
        gws = torch.empty(fa.load_library().fa_bwd_workspace_size(*gq.shape[:3]), dtype=torch.uint8,
                          device=dev)
        go, gl = fa.fa_fwd(gq, gk, gv, scale=w.softmax_scale, causal=True, stream=sptr)
        gdq, gdk, gdv = torch.empty_like(gq), torch.empty_like(gk), torch.empty_like(gv)
        ms = time_launches(lambda: fa.fa_bwd(gq, gk, gv, go, gl, gdo, scale=w.softmax_scale,
                                             causal=True, dq=gdq, dk=gdk, dv=gdv, stream=sptr,
                                             workspace=gws), flush, stream, n=5, warm=2)
        bflops = 2.5 * w.flops()
        backward["gqa_d256_causal"] = {
            "workload": w.name, "ms": round(ms, 4), "tflops": round(bflops / (ms * 1e-3) / 1e12, 1),
            "frac_of_peak": round(bflops / (ms * 1e-3) / 1e12 / peak, 3)}
        backward["flops"] = ("2.5 x the forward pass's (five GEMMs); three launches per call "
                             "(four at head_dim 256)")
        del gq, gk, gv, gdo, gws, go, gl, gdq, gdk, gdv
        assert fa.device_status(reset=True) == 0

    clk.section("bias")
    # ---- additive score bias on the bench workload: one [N, N] bias shared by all heads
    bias_line = {}
    if not args.no_bias:
        w = ws[0]  # non-causal pass
        g1 = torch.Generator(device=dev).manual_seed(2)
        bb = torch.randn((1, 1, w.Nq, w.Nk), device=dev, dtype=q.dtype, generator=g1)
        bo, bl = torch.empty_like(q), torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
        ms = time_launches(lambda: fa.fa_fwd(q, k, v, o=bo, lse=bl, scale=w.softmax_scale, bias=bb,
                                             stream=sptr), flush, stream)
        bias_line = {"workload": "LLaMA-7B layer non-causal + shared [N, N] fp16 bias",
                     **workload_line(w, ms, peak, hbm)}
        del bb, bo, bl
        assert fa.device_status(reset=True) == 0

    clk.section("window")
    # ---- sliding-window attention (causal, 1024-key window, 8192 positions, GQA 4)
    window = {}
    if not args.no_window:
        from fa_inputs import Workload
        ww = Workload("sliding window B2 Hq32 Hkv8 N8192 D128 fp16 causal, window 1024", 2, 32, 8,
                      8192, 8192, 128, "fp16", True, seed=0)
        W = 1024
        wq, wk, wv = (x.to(dev) for x in make_qkv(ww))
        wo, wl_ = torch.empty_like(wq), torch.empty(wq.shape[:3], dtype=torch.float32, device=dev)
        ms = time_launches(lambda: fa.fa_fwd(wq, wk, wv, o=wo, lse=wl_, scale=ww.softmax_scale,
                                             causal=True, window=(W - 1, -1), stream=sptr),
                           flush, stream)
        # visible (query, key) pairs per head: query i sees min(i + 1, W) keys
        pairs = W * (W + 1) // 2 + (ww.Nq - W) * W
        wflops = 4 * ww.B * ww.Hq * ww.D * pairs
        window = {"workload": ww.name, "visible_pairs_per_head": pairs,
                  **workload_line(ww, ms, peak, hbm, flops=wflops)}
        del wq, wk, wv, wo, wl_
        assert fa.device_status(reset=True) == 0

    clk.section("decode")
    # ---- KV-cache decode (one query row per head, long cache, GQA 4): HBM-bound
    decode = {}
    if not args.no_decode:
        from fa_inputs import Workload
        for wd in (Workload("decode B8 Hq32 Hkv8 Nq1 Nk32768 D128 fp16", 8, 32, 8, 1, 32768, 128,
                            "fp16", False, seed=0),
                   Workload("decode B1 Hq32 Hkv8 Nq1 Nk131072 D128 fp16", 1, 32, 8, 1, 131072,
                            128, "fp16", False, seed=0)):
            dq, dk, dv = (x.to(dev) for x in make_qkv(wd))
            do_, dl_ = torch.empty_like(dq), torch.empty(dq.shape[:3], dtype=torch.float32,
                                                         device=dev)
            # The K/V cache (>= 268 MB) is larger than L2, so launches run back to
            # back (no flush): a serving loop's view, with no host time between launches.
            for _ in range(3):
                fa.fa_fwd(dq, dk, dv, o=do_, lse=dl_, scale=wd.softmax_scale, stream=sptr)
            ts = []
            for i in range(5):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(10):
                    fa.fa_fwd(dq, dk, dv, o=do_, lse=dl_, scale=wd.softmax_scale, stream=sptr)
                b.record(stream)
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b) / 10)
            ms = statistics.median(ts)
            nbytes = wd.io_bytes()
            decode[wd.name] = {
                "ms": round(ms, 4), "bytes": nbytes,
                "l2": "K/V larger than L2, 10 launches back to back per event pair",
                "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                "frac_of_hbm": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 3),
                "tflops": round(wd.flops() / (ms * 1e-3) / 1e12, 2)}
            del dq, dk, dv, do_, dl_
        assert fa.device_status(reset=True) == 0

    clk.section("unfused")
    # ---- standard attention (the pages' comparison): S and P through device memory
    unfused = {}
    if not args.no_unfused:
        uws = torch.empty(int(fa.load_library().fa_fwd_unfused_workspace_size(*q.shape[:3], k.shape[2])),
                          dtype=torch.uint8, device=dev)
        uo, ul = torch.empty_like(q), torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
        for w in ws:
            ms = time_launches(lambda: fa.fa_fwd_unfused(q, k, v, o=uo, lse=ul, scale=w.softmax_scale,
                                                         causal=w.causal, stream=sptr,
                                                         workspace=uws), flush, stream)
            fused_ms = statistics.median(per_pass[ws.index(w)])
            n_scores = w.B * w.Hq * w.Nq * w.Nk
            unfused["causal" if w.causal else "non-causal"] = {
                "ms": round(ms, 4), "tflops": round(w.flops() / (ms * 1e-3) / 1e12, 1),
                "fused_ms": round(fused_ms, 4), "speedup_of_fused": round(ms / fused_ms, 2),
                "alg_bytes": w.io_bytes() + 12 * n_scores,
                "fused_alg_bytes": w.io_bytes()}
        unfused["alg_bytes_note"] = ("unfused: Q, K, V, O, LSE once plus S written and read (fp32) and "
                                     "P written and read (16-bit): 12 bytes per score; fused: none")
        unfused["workspace_bytes"] = uws.numel()
        del uws, uo, ul
        assert fa.device_status(reset=True) == 0

    clk.section("configs")
    # ---- every other workload the pages measure on, one line each (10 launches,
    # L2 flushed before each; the median).  Last: the long ones heat the GPU
    # into its power cap, which would slow the lines measured after them.
    from fa_inputs import TINY, LONG, gqa, seq_sweep
    configs = {}
    if not args.no_configs:
        cases = [("tiny B1 H1 N256 D64 fp16", TINY, None)]
        for n in (512, 2048, 4096, 8192):
            for causal in (False, True):
                cases.append((f"sweep B1 H32 N{n} D128 fp16 {'causal' if causal else 'non-causal'}",
                              seq_sweep(n, causal), None))
        for hkv, d in ((8, 128), (1, 128), (8, 64), (8, 256)):
            cases.append((f"gqa B4 Hq32 Hkv{hkv} N8192 D{d} bf16 causal", gqa(hkv, d), 11))
        cases.append(("long B1 Hq32 Hkv8 N131072 D128 bf16 causal, 1% outlier keys", LONG, 12))
        for name, w, dseed in cases:
            if dseed is None:
                cq, ck, cv = (x.to(dev) for x in make_qkv(w))
            else:
                cq, ck, cv = device_qkv(w, dev, dseed)
            co = torch.empty_like(cq)
            cl = torch.empty(cq.shape[:3], dtype=torch.float32, device=dev)
            n_launch = 3 if w.Nq > 65536 else 10
            ms = time_launches(lambda: fa.fa_fwd(cq, ck, cv, o=co, lse=cl, scale=w.softmax_scale,
                                                 causal=w.causal, stream=sptr),
                               flush, stream, n=n_launch, warm=2)
            configs[name] = workload_line(w, ms, peak, hbm)
            del cq, ck, cv, co, cl
        configs["note"] = ("ms: median CUDA-event time of one launch, L2 flushed before each; "
                           "alg_gbs: algorithmic bytes (read Q, K, V once, write O and LSE once) "
                           "per second, frac_of_hbm against the measured copy bandwidth")
        assert fa.device_status(reset=True) == 0
    gate = {}
    for n in (4096, 8192):
        for cz in ("non-causal", "causal"):
            c = configs.get(f"sweep B1 H32 N{n} D128 fp16 {cz}")
            if c:
                gate[f"N{n}_{cz.replace('-', '')}"] = {"ms": c["ms"], "tflops": c["tflops"],
                                                       "frac_of_peak": c["frac_of_peak"]}

    clk.__exit__(None, None, None)
    launch_ms = total_ms / world / (K * len(ws)) if world > 1 else total_ms / (K * len(ws))
    achieved = (flops_step / len(ws)) / (launch_ms * 1e-3) / 1e12
    traffic = recorded_traffic()
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(total_ms / K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp16",
        "data": "synthetic (seeded N(0,1), rounded to fp16; scale 1/sqrt(128))",
        "config": {"workload": "llama7b-attn B2 Hq32 Hkv32 N2048 D128 fp16, non-causal + causal",
                   "B": 2, "Hq": 32, "Hkv": 32, "N": 2048, "D": 128,
                   "passes_per_step": ["non-causal", "causal"],
                   "l2": "flushed before every pass (256 MiB write, outside the timed events)"},
        "per_pass": pass_lines,
        "pct_of_peak": {"measured_burst": round(100 * value / world / peak, 1),
                        "measured_sustained": round(100 * value / world / peak_sus, 1),
                        "spec_2250": round(100 * value / world / SPEC_PEAK_TFLOPS, 1),
                        "peak_source": peak_kind},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic,
                     "kernel": "fa::fa_fwd_kernel<128, 2, fp16> (D=128; the non-causal pass runs its "
                               "staged-epilogue instantiation)",
                     "peak_note": f"{peak_kind} bf16 dense burst (fp16:bf16 nominal ratio 1:1)"},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": "copies on their own streams, double-buffered: uploads and downloads "
                        "overlap the passes of the neighbouring steps"},
        "gpu_launches": K * len(ws),
        "clocks": clk.summary(),
        "configs": configs,
        "unfused": unfused,
        "gate_d128": gate,
        "decode": decode,
        "window": window,
        "backward": backward,
        "bias": bias_line,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        qkv = tuple(x for x in inputs[0][1:])
        f = s = 0.0
        reps = 0
        while s < 10.0 and reps < 64:  # about 10 s of wall time on all host cores
            df, ds = oracle_sample(ws, 512, reps, qkv)
            f, s, reps = f + df, s + ds, reps + 1
        line["cpu_baseline"] = {
            "value": f / s / 1e12, "unit": "TFLOP/s", "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": f"{reps} x 512 seeded query rows per (b, head) of each pass (non-causal, "
                      f"causal); {f / 1e9:.1f} GFLOP in {s:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

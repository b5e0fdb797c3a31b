"""Benchmark of the fused attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One step = one pass of the whole hot path over one batch of the LLaMA-7B
attention-layer workload (B=2, Hq=Hkv=32, N=2048, D=128, fp16,
scale=1/sqrt(128)): the non-causal forward pass and the causal forward pass,
both through the library's C ABI.  Inputs are synthetic (seeded N(0,1),
rounded to fp16) and resident in HBM when timing starts; L2 is flushed
(256 MiB write) between steps because the inputs (~100 MB) fit in L2.

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
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-gate", action="store_true", help="skip the N=4096/8192 gate configs")
    ap.add_argument("--no-decode", action="store_true", help="skip the KV-cache decode measurement")
    ap.add_argument("--no-window", action="store_true",
                    help="skip the sliding-window measurement")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward-pass measurement")
    ap.add_argument("--no-bias", action="store_true", help="skip the score-bias measurement")
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
    """NVML samples of SM clock and clock-event reasons while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int):
        self.ok = False
        self.samples, self.reasons = [], set()
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
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

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
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


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

    def step():
        for w, (o, lse) in zip(ws, outs):
            fa.fa_fwd(q, k, v, o=o, lse=lse, scale=w.softmax_scale, causal=w.causal, stream=sptr)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert fa.device_status(reset=True) == 0

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(ws) + 1)] for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(K):
            flush.zero_()
            e = ev[i]
            e[0].record(stream)
            for j, (w, (o, lse)) in enumerate(zip(ws, outs)):
                fa.fa_fwd(q, k, v, o=o, lse=lse, scale=w.softmax_scale, causal=w.causal,
                          stream=sptr)
                e[j + 1].record(stream)
        torch.cuda.synchronize()
    barrier()
    per_launch = [[ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K)] for j in range(len(ws))]
    step_ms = [sum(per_launch[j][i] for j in range(len(ws))) for i in range(K)]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    assert fa.device_status(reset=True) == 0
    flops_step = sum(w.flops() for w in ws)
    value = aggregate_tflops(flops_step, K, total_ms, world)

    # ---- end to end: pinned host inputs -> device -> both passes -> O and LSE back to host
    hq, hk, hv = (x.pin_memory() for x in inputs[0][1:])
    ho = [(torch.empty(q.shape, dtype=q.dtype, pin_memory=True),
           torch.empty(q.shape[:3], dtype=torch.float32, pin_memory=True)) for _ in ws]
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    d2h = sum(a.numel() * a.element_size() + b.numel() * b.element_size() for a, b in ho)
    qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    E = max(10, K // 20)

    def e2e_step():
        qd.copy_(hq, non_blocking=True)
        kd.copy_(hk, non_blocking=True)
        vd.copy_(hv, non_blocking=True)
        for w, (o, lse), (h_o, h_l) in zip(ws, outs, ho):
            fa.fa_fwd(qd, kd, vd, o=o, lse=lse, scale=w.softmax_scale, causal=w.causal, stream=sptr)
            h_o.copy_(o, non_blocking=True)
            h_l.copy_(lse, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = aggregate_tflops(flops_step, E, e2e_ms, world)

    # ---- gate configs (N = 4096 / 8192, D = 128), a few launches each, L2 flushed
    gate = {}
    if not args.no_gate:
        from fa_inputs import seq_sweep
        for n in (4096, 8192):
            w0 = seq_sweep(n, False)
            gq, gk, gv = (x.to(dev) for x in make_qkv(w0))
            go, gl = torch.empty_like(gq), torch.empty(gq.shape[:3], dtype=torch.float32, device=dev)
            for causal in (False, True):
                w = seq_sweep(n, causal)
                ts = []
                for i in range(13):
                    flush.zero_()
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    fa.fa_fwd(gq, gk, gv, o=go, lse=gl, scale=w.softmax_scale, causal=causal,
                              stream=sptr)
                    b.record(stream)
                    torch.cuda.synchronize()
                    if i >= 3:
                        ts.append(a.elapsed_time(b))
                ms = statistics.median(ts)
                gate[f"N{n}_{'causal' if causal else 'noncausal'}"] = {
                    "ms": round(ms, 4), "tflops": round(w.flops() / (ms * 1e-3) / 1e12, 1)}
            del gq, gk, gv, go, gl
        assert fa.device_status(reset=True) == 0

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
            ts = []
            for i in range(13):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fa.fa_bwd(q, k, v, bo, bl, bdo, scale=w.softmax_scale, causal=w.causal, dq=bdq,
                          dk=bdk, dv=bdv, stream=sptr, workspace=bws)
                b.record(stream)
                torch.cuda.synchronize()
                if i >= 3:
                    ts.append(a.elapsed_time(b))
            ms = statistics.median(ts)
            bflops = 2.5 * w.flops()  # five GEMMs against the forward pass's two
            backward["causal" if w.causal else "noncausal"] = {
                "ms": round(ms, 4), "tflops": round(bflops / (ms * 1e-3) / 1e12, 1),
                "frac_of_peak": round(bflops / (ms * 1e-3) / 1e12 / peaks()[0], 3)}
        backward["flops"] = "2.5 x the forward pass's (five GEMMs); three launches per call"
        del bdo, bws, bdq, bdk, bdv
        assert fa.device_status(reset=True) == 0

    # ---- additive score bias on the bench workload: one [N, N] bias shared by all heads
    bias_line = {}
    if not args.no_bias:
        w = ws[0]  # non-causal pass
        g1 = torch.Generator(device=dev).manual_seed(2)
        bb = torch.randn((1, 1, w.Nq, w.Nk), device=dev, dtype=q.dtype, generator=g1)
        bo, bl = torch.empty_like(q), torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
        ts = []
        for i in range(13):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fa.fa_fwd(q, k, v, o=bo, lse=bl, scale=w.softmax_scale, bias=bb, stream=sptr)
            b.record(stream)
            torch.cuda.synchronize()
            if i >= 3:
                ts.append(a.elapsed_time(b))
        ms = statistics.median(ts)
        bias_line = {"workload": "LLaMA-7B layer non-causal + shared [N, N] fp16 bias",
                     "ms": round(ms, 4), "tflops": round(w.flops() / (ms * 1e-3) / 1e12, 1),
                     "frac_of_peak": round(w.flops() / (ms * 1e-3) / 1e12 / peaks()[0], 3)}
        del bb, bo, bl
        assert fa.device_status(reset=True) == 0

    # ---- sliding-window attention (causal, 1024-key window, 8192 positions, GQA 4)
    window = {}
    if not args.no_window:
        from fa_inputs import Workload
        ww = Workload("sliding window B2 Hq32 Hkv8 N8192 D128 fp16 causal, window 1024", 2, 32, 8,
                      8192, 8192, 128, "fp16", True, seed=0)
        W = 1024
        wq, wk, wv = (x.to(dev) for x in make_qkv(ww))
        wo, wl_ = torch.empty_like(wq), torch.empty(wq.shape[:3], dtype=torch.float32, device=dev)
        ts = []
        for i in range(13):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fa.fa_fwd(wq, wk, wv, o=wo, lse=wl_, scale=ww.softmax_scale, causal=True,
                      window=(W - 1, -1), stream=sptr)
            b.record(stream)
            torch.cuda.synchronize()
            if i >= 3:
                ts.append(a.elapsed_time(b))
        ms = statistics.median(ts)
        # visible (query, key) pairs per head: query i sees min(i + 1, W) keys
        pairs = W * (W + 1) // 2 + (ww.Nq - W) * W
        wflops = 4 * ww.B * ww.Hq * ww.D * pairs
        window = {"workload": ww.name, "ms": round(ms, 4), "visible_pairs_per_head": pairs,
                  "tflops": round(wflops / (ms * 1e-3) / 1e12, 1),
                  "frac_of_peak": round(wflops / (ms * 1e-3) / 1e12 / peaks()[0], 3)}
        del wq, wk, wv, wo, wl_
        assert fa.device_status(reset=True) == 0

    # ---- KV-cache decode (one query row per head, 32K-token cache, GQA 4): HBM-bound
    decode = {}
    if not args.no_decode:
        from fa_inputs import Workload
        wd = Workload("decode B8 Hq32 Hkv8 Nq1 Nk32768 D128 fp16", 8, 32, 8, 1, 32768, 128, "fp16",
                      False, seed=0)
        dq, dk, dv = (x.to(dev) for x in make_qkv(wd))
        do_, dl_ = torch.empty_like(dq), torch.empty(dq.shape[:3], dtype=torch.float32, device=dev)
        # The K/V cache (1.07 GB) is 8x the L2, so launches run back to back (no
        # flush): a serving loop's view, with no host time between launches.
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
        hbm = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["hbm_gbs"] \
            if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else 6650.0
        decode = {"workload": wd.name, "ms": round(ms, 4), "bytes": nbytes,
                  "l2": "inputs larger than L2 (1.07 GB K/V), 10 launches back to back per event pair",
                  "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                  "frac_of_hbm": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 3),
                  "tflops": round(wd.flops() / (ms * 1e-3) / 1e12, 2)}
        del dq, dk, dv, do_, dl_
        assert fa.device_status(reset=True) == 0

    peak, peak_sus, peak_kind = peaks()
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
                   "l2": "flushed between steps (256 MiB write, outside the timed events)"},
        "pct_of_peak": {"measured_burst": round(100 * value / world / peak, 1),
                        "measured_sustained": round(100 * value / world / peak_sus, 1),
                        "spec_2250": round(100 * value / world / SPEC_PEAK_TFLOPS, 1),
                        "peak_source": peak_kind},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic,
                     "kernel": "fa::fa_fwd_kernel<128, 2, false> (fp16, D=128)",
                     "peak_note": f"{peak_kind} bf16 dense burst (fp16:bf16 nominal ratio 1:1)"},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": K * len(ws),
        "clocks": clk.summary(),
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

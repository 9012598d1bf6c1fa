#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200: one step = the forward
(O and LSE) plus the backward (dQ, dK, dV) over one batch of synthetic input.

Default workload: the largest stated single-GPU problem, head_dim 256 with GQA
ratio 8 (8 query heads, 1 key-value head) over one 131072-token sequence,
non-causal, bf16 N(0,1) (the "FA4 head_dim=256 B200 Regression Check" shape
lists).  ``--workload varlen_gqa`` selects the packed varlen GQA batch of the
cosmos-framework issue #118 benchmark (16384 tokens in segments of 128..4096,
32 query / 8 key-value heads, head_dim 128), and the other names below the
rest of the stated shapes.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the fp64 CPU oracle as the reference arm

Prints one JSON line (rank 0).  FLOPs follow the pages: forward 4*s_q*s_k*H*D per
segment (halved when causal), forward+backward 3.5x that, backward alone 2.5x.
Multi-GPU runs (torchrun) are independent replicas: the path has no exchange
step, so no collective touches the data; ranks only meet for the timing barrier
and the max-over-ranks reduction.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth_inputs as si  # noqa: E402

PAGE_PEAK_TFLOPS = 2250.0  # B200 dense bf16 peak as the FA4 hd256 regression check states it
L2_FLUSH_BYTES = 512 << 20
METRIC = "attention fwd & fwd+bwd TFLOP/s (bf16) and % of B200 dense bf16 peak"

WORKLOADS = {
    "varlen_gqa": lambda: si.varlen_gqa(),
    "gqa_16k": lambda: si.single_gqa(16384),
    "gqa_16k_causal": lambda: si.single_gqa(16384, True),
    "gqa_64k": lambda: si.single_gqa(65536),
    "d64_mha": lambda: si.d64_mha(),
    "d256_mha_16k": lambda: si.d256_mha(16384, False),
    "d256_mha_16k_causal": lambda: si.d256_mha(16384, True),
    "d256_gqa8_128k": lambda: si.d256_gqa8(131072, False),
    "d256_gqa8_128k_causal": lambda: si.d256_gqa8(131072, True),
    "gqa_16k_swa": lambda: si.gqa_sliding_window(16384, 4096),
    "decode_64x64k": lambda: si.decode_gqa(64, 65536),
    "gqa_16k_softcap": lambda: si.gqa_softcap(16384, 50.0),
    "tiny": lambda: si.tiny(),
    "varlen_short": lambda: si.short_segments(128, 16384),
}
# the rest of the pages' shape lists: GQA head_dim 128 single segments
# (1K/4K/32K; 16K and 64K above) and head_dim 256 MHA with 8 heads at batch
# 8/4/2/1 x 4K/8K/16K/32K and batch 1 at 64K/128K, causal and not
for _s in (1024, 4096, 32768):
    WORKLOADS[f"gqa_{_s // 1024}k"] = (lambda s=_s: si.single_gqa(s))
for _s in (4096, 8192, 32768, 65536, 131072):
    WORKLOADS[f"d256_mha_{_s // 1024}k"] = (lambda s=_s: si.d256_mha(s, False))
    WORKLOADS[f"d256_mha_{_s // 1024}k_causal"] = (lambda s=_s: si.d256_mha(s, True))
# head_dim 256 GQA ratio 8 at the shorter lengths of the same shape list (one
# sequence each; the stated problem is the 128K one above)
for _s in (4096, 8192, 16384, 32768, 65536):
    WORKLOADS[f"d256_gqa8_{_s // 1024}k"] = (lambda s=_s: si.d256_gqa8(s, False))
    WORKLOADS[f"d256_gqa8_{_s // 1024}k_causal"] = (lambda s=_s: si.d256_gqa8(s, True))


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}, "fallback"


def strip_c_comments(text: str) -> str:
    """C/C++ source without its comments and with runs of blank space collapsed,
    so that edits to comments alone do not change the source hash.  String and
    character literals are kept as they are."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


# the sources each timed kernel is compiled from (the C ABI file launches both)
KERNEL_SOURCES = {
    "attn_fwd": ("api.cu", "ptx.cuh", "fwd_kernel.cuh", "fwd_pair_kernel.cuh"),
    "attn_bwd_main": ("api.cu", "ptx.cuh", "bwd_kernels.cuh", "bwd_pair_kernel.cuh"),
}


def library_source_hash(kernel: str | None = None):
    """Hash of a kernel's sources (all kernel and ABI sources when kernel is None)
    with comments removed: a recorded ncu traffic figure stays valid across
    comment edits and edits of other kernels, not across edits of its own code."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_attention_129_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) if kernel else None
    for name in sorted(os.listdir(csrc)):
        if not name.endswith((".cu", ".cuh", ".h")) or (names and name not in names):
            continue
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode())
            h.update(strip_c_comments(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the
    current kernel sources; otherwise None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{kernel}/{workload}")
    if not e or e.get("source_hash") != library_source_hash(kernel):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.05):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as e:  # no NVML: report what is missing instead of clocks
            self.error = str(e)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.error}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        if world == 1 and n_gpus > 1:
            raise SystemExit("--gpus N > 1 must be launched with torchrun (one rank per GPU)")
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int, dev) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    # NCCL reduces device tensors; the gloo backend (CPU tests) host tensors
    where = dev if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=where)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline arm; the oracle is never on the product path)
# ---------------------------------------------------------------------------
def oracle_sample(wl: si.Workload, seconds: float):
    """A bounded sample of the workload for the oracle: whole segments taken in
    order, one key/value head group, grown until the estimated time is
    `seconds`.  Returns (sample workload, description)."""
    import oracle
    G = wl.hq // wl.hkv
    # calibrate the oracle's rate on a 256-token segment of this head group
    cal = si.Workload("cal", [256], G, 1, wl.d, wl.causal, seed=wl.seed, window=wl.window,
                      softcap=wl.softcap)
    q, k, v, do = cal.tensors()
    t0 = time.perf_counter()
    oracle.fwd(q, k, v, cal.cu_q, cal.cu_k, cal.scale, cal.causal, window=cal.window,
               softcap=cal.softcap)
    oracle.bwd(q, k, v, do, cal.cu_q, cal.cu_k, cal.scale, cal.causal, window=cal.window,
               softcap=cal.softcap)
    rate = 3.5 * cal.fwd_flops() / max(time.perf_counter() - t0, 1e-6)
    lengths = []
    budget = seconds * rate
    for s in wl.lengths_q:
        trial = lengths + [s]
        f = 3.5 * si.Workload("t", trial, G, 1, wl.d, wl.causal, window=wl.window).fwd_flops()
        if lengths and f > budget:
            break
        lengths = trial
        if f > budget:
            break
    if len(lengths) == 1 and 3.5 * si.Workload("t", lengths, G, 1, wl.d, wl.causal,
                                                window=wl.window).fwd_flops() > 4 * budget:
        # one segment is far over budget: take a shorter prefix of it
        s = int(np.sqrt(budget / (3.5 * 4 * G * wl.d * (0.5 if wl.causal else 1.0))))
        lengths = [max(64, s)]
    sample = si.Workload(f"{wl.name}_oracle_sample", lengths, G, 1, wl.d, wl.causal, seed=wl.seed,
                         window=wl.window, softcap=wl.softcap)
    desc = (f"{len(lengths)} segment(s) {lengths[:6]}{'...' if len(lengths) > 6 else ''} "
            f"of the workload, {G} query heads / 1 key-value head, head_dim {wl.d}, "
            f"{'causal' if wl.causal else 'non-causal'}: full oracle forward + backward")
    return sample, desc


def time_oracle(sample: si.Workload):
    import oracle
    q, k, v, do = sample.tensors()
    t0 = time.perf_counter()
    oracle.fwd(q, k, v, sample.cu_q, sample.cu_k, sample.scale, sample.causal,
               window=sample.window, softcap=sample.softcap)
    oracle.bwd(q, k, v, do, sample.cu_q, sample.cu_k, sample.scale, sample.causal,
               window=sample.window, softcap=sample.softcap)
    return time.perf_counter() - t0


def host_cpu():
    """The host's CPU model and its logical and physical core counts."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        import psutil
        physical = psutil.cpu_count(logical=False)
    except Exception:
        physical = None
    return {"cpu_model": model, "logical_cores": os.cpu_count(), "physical_cores": physical}


def cpu_baseline(wl, seconds=15.0):
    import oracle
    sample, desc = oracle_sample(wl, seconds)
    dt = time_oracle(sample)
    rate = 3.5 * sample.fwd_flops() / dt  # FLOP/s of the oracle on this sample
    return {"value": rate / 1e12, "unit": "TFLOP/s",
            "cores": oracle.num_threads(), "kind": "oracle", "sample": desc,
            "seconds": round(dt, 2),
            # the whole workload at the sample's rate (extrapolated, not run)
            "full_workload_seconds_extrapolated": round(3.5 * wl.fwd_flops() / rate, 1),
            **host_cpu()}


def run_reference(args, wl, world, rank):
    """The reference arm: the fp64 CPU oracle, timed step by step on a bounded
    sample of the same workload (rank 0 only)."""
    if rank != 0:
        return None
    import oracle
    per_step = max(0.05, min(5.0, 150.0 / max(1, args.steps + args.warmup)))
    sample, desc = oracle_sample(wl, per_step)
    for _ in range(args.warmup):
        time_oracle(sample)
    times = [time_oracle(sample) for _ in range(args.steps)]
    total = sum(times)
    value = 3.5 * sample.fwd_flops() * args.steps / total / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, "none (CPU)"),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": desc, **host_cpu()},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def config_of(wl, l2, num_splits=1):
    return {"workload": wl.name, "segments": len(wl.lengths_q), "total_tokens": wl.total_q,
            "total_keys": wl.total_k, "num_splits": num_splits,
            "nheads_q": wl.hq, "nheads_kv": wl.hkv, "head_dim": wl.d, "causal": wl.causal,
            "window": list(wl.window) if wl.window is not None else None,
            "softcap": wl.softcap or None,
            "softmax_scale": wl.scale, "l2": l2, "parallelism": "replicas"}


def fwd_lse_on_off(ea, wl, q, k, v, cu_q, cu_k, out, lse, dev, rounds=8, calls=8):
    """The forward alone with return_lse on and off (the head_dim-64 config asks
    that both reach the same throughput class).  After about a second of bf16
    matmuls to bring the clocks up, each arm is a CUDA graph of `calls` forward
    calls, replayed in rounds that alternate which arm goes first, so clock drift
    under the power cap falls on both arms alike; medians over the rounds."""
    a = torch.randn(8192, 8192, device=dev, dtype=torch.bfloat16)
    t0 = time.time()
    while time.time() - t0 < 1.0:
        for _ in range(8):
            torch.mm(a, a)
        torch.cuda.synchronize()
    del a
    graphs = {}
    for rl in (True, False):
        def fwd(rl=rl):
            ea.attn_fwd(q, k, v, cu_q, cu_k, wl.max_q, wl.max_k, scale=wl.scale,
                        causal=wl.causal, window=wl.window, softcap=wl.softcap,
                        return_lse=rl, out=out, lse=lse if rl else None)
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(2):
                fwd()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(calls):
                fwd()
        graphs[rl] = g
    times = {True: [], False: []}
    for r in range(rounds):
        for rl in ((True, False) if r % 2 == 0 else (False, True)):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graphs[rl].replay()
            e1.record()
            torch.cuda.synchronize()
            times[rl].append(e0.elapsed_time(e1) / calls)
    rc, msg = ea.last_device_error()
    if rc != 0:
        raise RuntimeError(f"device error in the return_lse comparison: {msg}")
    F = wl.fwd_flops()
    on, off = statistics.median(times[True]), statistics.median(times[False])
    return {"lse_on_tflops": F / (on * 1e-3) / 1e12, "lse_off_tflops": F / (off * 1e-3) / 1e12,
            "off_over_on": on / off, "rounds": rounds, "calls_per_graph": calls,
            "method": "CUDA-graph replay, alternating order, 1 s matmul warm-up, medians"}


SUSTAINED_AFTER_S = 1.0  # timed regions at least this long are held to the sustained peak


def kernel_rooflines(wl, fwd_ms, bwd_main_ms, peaks, peak_kind, timed_s):
    """Per kernel: algorithmic FLOPs (the pages' convention: the backward is
    2.5x the forward) and the bytes the method must move, over the live
    CUDA-event time, with the roof that binds at that arithmetic intensity;
    and the roofline object of the dominant kernel (the one that takes longer)
    against the measured peak of its bound.

    Which matmul peak: the burst figure (best of short cuBLAS runs) for kernels
    timed in a short region, the sustained one (seconds of back-to-back GEMMs
    under the power cap) when the timed region runs ``SUSTAINED_AFTER_S`` or
    longer.  The fraction of the other one is reported beside it."""
    F = wl.fwd_flops()
    burst = peaks.get("bf16_tflops", 1590.0)
    sustained = peaks.get("bf16_tflops_sustained", 1400.0)
    long_region = timed_s >= SUSTAINED_AFTER_S
    peak = sustained if long_region else burst
    peak_bw = peaks.get("hbm_gbs", 6650.0)
    kernels = {}
    for kname, kflops, kbytes, kms in (("attn_fwd", F, wl.fwd_bytes(True), fwd_ms),
                                      ("attn_bwd_main", 2.5 * F, wl.bwd_main_bytes(),
                                       bwd_main_ms)):
        kernels[kname] = {
            "ms_per_launch": kms, "algorithmic_flops_per_launch": kflops,
            "algorithmic_bytes_per_launch": kbytes,
            "tflops": kflops / (kms * 1e-3) / 1e12, "gbs": kbytes / (kms * 1e-3) / 1e9,
            "bound": "hbm" if kbytes / peak_bw > kflops / (peak * 1e3) else "tensor"}
    kname = "attn_bwd_main" if bwd_main_ms >= fwd_ms else "attn_fwd"
    kd = kernels[kname]
    if kd["bound"] == "tensor":
        roofline = {"bound": "tensor", "achieved": kd["tflops"], "peak": peak,
                    "unit": "TFLOP/s", "frac": kd["tflops"] / peak,
                    "peak_kind": (f"{peak_kind} {'sustained' if long_region else 'burst'} "
                                  f"bf16 matmul (timed region {timed_s:.2f} s)"),
                    "frac_of_burst": kd["tflops"] / burst,
                    "frac_of_sustained": kd["tflops"] / sustained}
    else:
        roofline = {"bound": "hbm", "achieved": kd["gbs"], "peak": peak_bw, "unit": "GB/s",
                    "frac": kd["gbs"] / peak_bw, "peak_kind": f"{peak_kind} HBM copy"}
    roofline.update({"kernel": kname, "traffic": None,
                     "algorithmic_flops_per_launch": kd["algorithmic_flops_per_launch"],
                     "algorithmic_bytes_per_launch": kd["algorithmic_bytes_per_launch"],
                     "ms_per_launch": kd["ms_per_launch"]})
    return kernels, roofline


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, wl, world, rank, local):
    import exact_attention_129_b200 as ea
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    q_h, k_h, v_h, do_h = wl.tensors()
    cu_q_h = torch.from_numpy(wl.cu_q)
    cu_k_h = torch.from_numpy(wl.cu_k)
    q, k, v, do = (t.to(dev) for t in (q_h, k_h, v_h, do_h))
    cu_q, cu_k = cu_q_h.to(dev), cu_k_h.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((wl.hq, wl.total_q), device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(ea.bwd_workspace_size(len(wl.lengths_q), wl.total_q, wl.hq, wl.d),
                     device=dev, dtype=torch.uint8)
    fws = None
    if args.num_splits > 1:
        fws = torch.empty(ea.fwd_split_workspace_size(wl.total_q, wl.hq, wl.d, args.num_splits),
                          device=dev, dtype=torch.uint8)
    flush = torch.empty(L2_FLUSH_BYTES, device=dev, dtype=torch.uint8)
    F = wl.fwd_flops()

    def step():
        ea.attn_fwd(q, k, v, cu_q, cu_k, wl.max_q, wl.max_k, scale=wl.scale, causal=wl.causal,
                    window=wl.window, softcap=wl.softcap, return_lse=True, out=out, lse=lse,
                    num_splits=args.num_splits, workspace=fws)
        ea.attn_bwd(q, k, v, out, lse, do, cu_q, cu_k, wl.max_q, wl.max_k, scale=wl.scale,
                    causal=wl.causal, window=wl.window, softcap=wl.softcap, dq=dq, dk=dk, dv=dv,
                    workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    rc, msg = ea.last_device_error()
    if rc != 0:
        raise RuntimeError(f"device error during warm-up: {msg}")

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    s_ev = [(ev(), ev()) for _ in range(args.steps)]
    f_ev = [(ev(), ev()) for _ in range(args.steps)]
    b_ev = [(ev(), ev()) for _ in range(args.steps)]
    for a, b in f_ev + b_ev:  # torch creates the CUDA event on first record
        a.record()
        b.record()
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        for i in range(args.steps):
            flush.zero_()  # evict L2 between steps (outside the timed events)
            ea.set_timing_events(ea.KERNEL_FWD, *f_ev[i])
            ea.set_timing_events(ea.KERNEL_BWD_MAIN, *b_ev[i])
            s_ev[i][0].record()
            step()
            s_ev[i][1].record()
        torch.cuda.synchronize()
    ea.set_timing_events(ea.KERNEL_FWD)
    ea.set_timing_events(ea.KERNEL_BWD_MAIN)
    barrier(world)
    rc, msg = ea.last_device_error()
    if rc != 0:
        raise RuntimeError(f"device error in the timed region: {msg}")
    step_ms = sum(a.elapsed_time(b) for a, b in s_ev)
    fwd_ms = sum(a.elapsed_time(b) for a, b in f_ev) / args.steps
    bwd_main_ms = sum(a.elapsed_time(b) for a, b in b_ev) / args.steps
    total_ms = max_over_ranks(step_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = world * 3.5 * F * args.steps / (total_ms * 1e-3) / 1e12

    # end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e:
        hq_, hk_, hv_, hdo = (t.pin_memory() for t in (q_h, k_h, v_h, do_h))
        hcq, hck = cu_q_h.pin_memory(), cu_k_h.pin_memory()
        h_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        h_lse = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        h_dq = torch.empty(dq.shape, dtype=dq.dtype, pin_memory=True)
        h_dk = torch.empty(dk.shape, dtype=dk.dtype, pin_memory=True)
        h_dv = torch.empty(dv.shape, dtype=dv.dtype, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in (hq_, hk_, hv_, hdo, hcq, hck))
        d2h = sum(t.numel() * t.element_size() for t in (h_out, h_lse, h_dq, h_dk, h_dv))
        n_e2e = max(3, min(args.steps, 20))

        def e2e_step():
            for d_, h_ in ((q, hq_), (k, hk_), (v, hv_), (do, hdo), (cu_q, hcq), (cu_k, hck)):
                d_.copy_(h_, non_blocking=True)
            step()
            for h_, d_ in ((h_out, out), (h_lse, lse), (h_dq, dq), (h_dk, dk), (h_dv, dv)):
                h_.copy_(d_, non_blocking=True)

        for _ in range(2):
            e2e_step()
        e_ev = [(ev(), ev()) for _ in range(n_e2e)]
        barrier(world)
        torch.cuda.synchronize()
        for i in range(n_e2e):
            flush.zero_()
            e_ev[i][0].record()
            e2e_step()
            e_ev[i][1].record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in e_ev), world, dev)
        e2e = {"value": world * 3.5 * F * n_e2e / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "ms_per_step": e_ms / n_e2e}

    peaks, peak_kind = measured_peaks()
    kernels, roofline = kernel_rooflines(wl, fwd_ms, bwd_main_ms, peaks, peak_kind,
                                         total_ms * 1e-3)
    roofline["traffic"] = recorded_traffic(roofline["kernel"], wl.name)

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16; varlen lengths seeded uniform)",
        "config": config_of(wl, "flushed between steps (512 MiB write)", args.num_splits),
        "fwd_tflops": F / (fwd_ms * 1e-3) / 1e12,
        "fwd_ms": fwd_ms, "bwd_main_ms": bwd_main_ms,
        "pct_of_2250": {"fwd": 100 * F / (fwd_ms * 1e-3) / 1e12 / PAGE_PEAK_TFLOPS,
                        "fwd_bwd": 100 * value / world / PAGE_PEAK_TFLOPS},
        "pct_of_measured_burst": {
            "fwd": 100 * F / (fwd_ms * 1e-3) / 1e12 / peaks.get("bf16_tflops", 1590.0),
            "fwd_bwd": 100 * value / world / peaks.get("bf16_tflops", 1590.0)},
        "roofline": roofline,
        "kernels": kernels,
        "clocks": sampler.summary(),
        "e2e": e2e,
        # per step: forward (+ SplitKV combine), backward preprocess, main and,
        # unless every key segment fits one 128-key block (dQ stored directly),
        # the dQ convert
        "gpu_launches": ((2 if args.num_splits > 1 else 1) + 2
                         + (0 if wl.max_k <= 128 and os.environ.get("ATTN_BWD_DQ_DIRECT") != "0"
                            else 1)) * args.steps,
        "library": ea.library().attn_version().decode(),
    }
    if args.lse_ab or args.workload == "d64_mha":
        line["fwd_lse_on_off"] = fwd_lse_on_off(ea, wl, q, k, v, cu_q, cu_k, out, lse, dev)
    return line


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="d256_gqa8_128k")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--num-splits", type=int, default=1,
                    help="SplitKV parts of the forward (1: plain forward)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--lse-ab", action="store_true",
                    help="also time the forward alone with return_lse on and off "
                         "(always done for the d64_mha workload)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    wl = WORKLOADS[args.workload]()

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, wl, int(os.environ.get("WORLD_SIZE", "1")), rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    world, rank, local = dist_setup(args.gpus)
    try:
        line = run_ours(args, wl, world, rank, local)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
            else:
                line["cpu_baseline"] = None
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Benchmark of the SageAttention forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sage|reference]
                    [--workload NAME] [--extra-workloads a,b] [--no-e2e] [--no-cpu-baseline]

A step is one pass of the whole path over one batch of synthetic input:
sage_quant_qkv (smooth K / smooth Q + delta_S, INT8 Q/K, FP8 V) followed by
the fused INT8/FP8 attention kernel.  The metric is attention TOPS
(4 N^2 d per head, halved when causal).  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (the plain scalar reference of the
method) on a bounded sample of the same workload on the host cores.
Multi-GPU (torchrun): every rank runs the same per-GPU workload (weak
scaling, no collective on the data path); time = max over ranks.
"""
from __future__ import annotations

import argparse
import faulthandler
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

_ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, _ROOT)

from quantized_attention_block_b200 import workloads as W  # noqa: E402

INT8_FP8_PER_BF16 = 2.0  # nominal dense ratio 4.5 / 2.25 PFLOP/s
FP4_PER_BF16 = 4.0  # nominal dense ratio 9 / 2.25 PFLOP/s


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one attention
# launch of the prefill workload: one ncu capture of attn_i8f8_kernel at B=3
# (431.9 + 69.2 MB), scaled to B=4 by the number of heads.  Valid only for the
# kernel sources it was taken on (hash below); any other source reports null.
ATTN_TRAFFIC = {"bytes": (431864064 + 69236480) * 4 / 3, "src_sha256_16": "d608e0ce163c0c7c",
                "workload": "llm_prefill_causal_B4_H32_N4096_d128"}


def _attn_src_sha() -> str:
    """Hash of the sources that decide the attention kernel's memory traffic."""
    import hashlib
    h = hashlib.sha256()
    for name in ("attn_i8f8.cu", "common.cuh"):
        with open(os.path.join(_ROOT, "quantized_attention_block_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _attn_traffic(w: W.Workload):
    sha = _attn_src_sha()
    if sha != ATTN_TRAFFIC["src_sha256_16"] or w.name != ATTN_TRAFFIC["workload"]:
        return None
    return ATTN_TRAFFIC["bytes"]


def _peaks():
    path = os.path.join(_ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


_SAMPLER_CODE = r"""
import sys, time
import pynvml as nv
nv.nvmlInit()
try:
    h = nv.nvmlDeviceGetHandleByPciBusId(sys.argv[1])
except Exception:
    h = nv.nvmlDeviceGetHandleByIndex(int(sys.argv[3]))
period = float(sys.argv[2])
print("max", nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM), flush=True)
while True:
    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
    try:
        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
    except Exception:
        rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
    pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
    print(time.monotonic_ns(), sm, rs, pw, flush=True)
    time.sleep(period)
"""


class ClockSampler:
    """Samples SM clock, power and clock-event (throttle) reasons through NVML
    every few milliseconds from a separate process (its own interpreter, so the
    launching thread cannot starve it), time-stamped with the system monotonic
    clock.  mark() brackets a region; summary() reports the samples inside the
    marked regions."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device: int, period_s: float = 0.002):
        self.dev = torch_device
        self.period = period_s
        self.samples = []
        self.regions = {}
        self.err = None
        self.proc = None
        self.max_sm = None

    def __enter__(self):
        try:
            props = torch.cuda.get_device_properties(self.dev)
            bus = "%08X:%02X:%02X.0" % (int(props.pci_domain_id), int(props.pci_bus_id), int(props.pci_device_id))
            self.proc = subprocess.Popen([sys.executable, "-c", _SAMPLER_CODE, bus, str(self.period), str(self.dev)],
                                         stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
            first = self.proc.stdout.readline().split()
            if len(first) != 2 or first[0] != "max":
                raise RuntimeError("sampler did not start: " + self.proc.stderr.read()[-300:])
            self.max_sm = int(first[1])
            # one sample before the caller's region starts (a short region may
            # otherwise end before the first sample)
            f = self.proc.stdout.readline().split()
            if len(f) == 4:
                self.samples.append((int(f[0]), int(f[1]), int(f[2]), float(f[3])))
        except Exception as e:  # pragma: no cover
            self.err = f"nvml unavailable: {e}"
            self.proc = None
        return self

    def mark(self, name: str, begin: bool):
        t = time.monotonic_ns()
        if begin:
            self.regions[name] = [t, None]
        else:
            self.regions[name][1] = t

    def __exit__(self, *exc):
        if self.proc is None:
            return
        time.sleep(3 * self.period)
        self.proc.kill()
        out, _ = self.proc.communicate(timeout=5)
        for ln in out.splitlines():
            f = ln.split()
            if len(f) == 4:
                self.samples.append((int(f[0]), int(f[1]), int(f[2]), float(f[3])))

    def summary(self, region: str = "timed"):
        if self.proc is None and not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err or "no samples"]}
        t0, t1 = self.regions.get(region, [0, 1 << 62])
        inside = [x for x in self.samples if t0 <= x[0] <= t1]
        if not inside:
            # no sample landed in a very short region: the one just before it
            before = [x for x in self.samples if x[0] < t0]
            inside = before[-1:]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_sm, "reasons": ["no samples"]}
        sm = [x[1] for x in inside]
        reasons = sorted({name for _, _, rs, _ in inside for bit, name in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_sm, "sm_min_mhz": min(sm),
                "reasons": reasons, "samples": len(inside), "region_ms": (t1 - t0) / 1e6,
                "power_w_max": max(x[3] for x in inside), "source": "nvml (separate process, 2 ms period)"}


def _barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def _max_over_ranks(x: float, ws: int) -> float:
    """The largest of the ranks' values (device time of the slowest rank)."""
    if ws == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_tops(ops_per_rank: float, ms_max: float, ws: int) -> float:
    """Whole-job throughput: every rank processes one copy of the workload (its
    own seeded inputs), the job takes as long as the slowest rank."""
    return ws * ops_per_rank / (ms_max * 1e-3) / 1e12


def rank_seed(w: W.Workload, rank: int) -> int:
    """Each rank draws its own inputs of the same shape (weak scaling)."""
    return w.seed + rank


def pv_mode(w: W.Workload, choice: str) -> int:
    """auto: the two-level scheme where the workload's recipe names it, else the
    TMEM FP32 accumulator (tcgen05 accumulates FP8 products in full FP32)."""
    if choice == "auto":
        return 0 if w.names_two_level else 1
    return {"two_level": 0, "tmem_fp32": 1}[choice]


def run_sage(w: W.Workload, steps: int, warmup: int, ws: int, rank: int, local: int, e2e: bool,
             pv_accum: int = 0, time_other_mode: bool = False):
    from quantized_attention_block_b200 import sage

    q, k, v = W.make_qkv(w, seed=rank_seed(w, rank))
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    p = sage.make_params(qd, kd, causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k,
                         smooth_q=w.smooth_q, bq=w.bq, bk=w.bk, pv_accum=pv_accum)
    wsp = sage.alloc_nvfp4_workspace(p) if w.nvfp4 else sage.alloc_workspace(p)
    o = torch.empty_like(qd)
    stream = torch.cuda.current_stream()
    quant = sage.sage_quant_nvfp4 if w.nvfp4 else sage.sage_quant_qkv
    attn = sage.sage_attn_fwd_nvfp4_quantized if w.nvfp4 else sage.sage_attn_fwd_quantized
    if w.nvfp4:
        time_other_mode = False  # one accumulation scheme on the NVFP4 path

    def step(ev=None):
        view = quant(qd, kd, vd, p, wsp, stream)
        if ev is not None:
            ev[0].record(stream)
        attn(view, o, p, stream)
        if ev is not None:
            ev[1].record(stream)

    for _ in range(max(3, warmup)):
        step()
    torch.cuda.synchronize()
    # our kernels per step: the quantisation kernels (as the library reports
    # them for the path the sizes take) + the attention
    n_quant = sage.sage_quant_nvfp4_kernel_count(p) if w.nvfp4 else sage.sage_quant_kernel_count(p)
    launches_per_step = n_quant + 1
    attn_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        _barrier(ws)
        torch.cuda.synchronize()
        clk.mark("timed", True)
        t0.record(stream)
        for i in range(steps):
            step(attn_ev[i])
        t1.record(stream)
        torch.cuda.synchronize()
        clk.mark("timed", False)
        _barrier(ws)
    ms_total = t0.elapsed_time(t1)
    ms_attn = sum(a.elapsed_time(b) for a, b in attn_ev) / steps
    assert sage.sage_last_device_error() == 0
    ms_step = _max_over_ranks(ms_total / steps, ws)
    ms_attn = _max_over_ranks(ms_attn, ws)
    res = {"ms_step": ms_step, "ms_attn": ms_attn, "ms_quant": ms_step - ms_attn, "clocks": clk.summary(),
           "gpu_launches": launches_per_step * steps}
    if time_other_mode:
        # kernel time of the other P~V accumulation mode on the same inputs (for the record)
        p2 = sage.make_params(qd, kd, causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k,
                              smooth_q=w.smooth_q, bq=w.bq, bk=w.bk, pv_accum=1 - pv_accum)
        view = sage.sage_quant_qkv(qd, kd, vd, p2, wsp, stream)
        for _ in range(3):
            sage.sage_attn_fwd_quantized(view, o, p2, stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = max(3, steps // 2)
        e0.record(stream)
        for _ in range(n):
            sage.sage_attn_fwd_quantized(view, o, p2, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        res["ms_attn_other_mode"] = _max_over_ranks(e0.elapsed_time(e1) / n, ws)

    if e2e:
        # End to end through the public one-call API, pipelined over steps the
        # way a serving loop runs it: device inputs and outputs are double
        # buffered; step i's host->device copies (copy stream) overlap step
        # i-1's attention (compute stream) and step i-2's device->host read of
        # the output (read-back stream).  Every step copies its own inputs from
        # pinned host memory and reads its own output back.
        qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
        ohs = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for _ in range(2)]
        bufs = [(qd, kd, vd, o), (torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd),
                                  torch.empty_like(o))]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer b landed
        ev_used = [torch.cuda.Event() for _ in range(2)]  # attention done with buffer b
        ev_out = [torch.cuda.Event() for _ in range(2)]   # output of buffer b read back

        def e2e_step(i):
            b = i % 2
            qb, kb, vb, ob = bufs[b]
            s_in.wait_event(ev_used[b])  # the attention of step i-2 has read buffer b
            with torch.cuda.stream(s_in):
                qb.copy_(qh, non_blocking=True)
                kb.copy_(kh, non_blocking=True)
                vb.copy_(vh, non_blocking=True)
            ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])  # step i-2's output has been read back
            if w.nvfp4:
                sage.sage_attn_fwd_nvfp4(qb, kb, vb, causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k,
                                         smooth_q=w.smooth_q, bq=w.bq, out=ob, workspace=wsp, stream=stream)
            else:
                sage.sage_attn_fwd(qb, kb, vb, causal=w.causal, sm_scale=w.sm_scale, smooth_k=w.smooth_k,
                                   smooth_q=w.smooth_q, bq=w.bq, bk=w.bk, pv_accum=pv_accum, out=ob,
                                   workspace=wsp, stream=stream)
            ev_used[b].record(stream)
            s_out.wait_event(ev_used[b])
            with torch.cuda.stream(s_out):
                ohs[b].copy_(ob, non_blocking=True)
            ev_out[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        e_steps = max(3, steps)  # the same K steps as the device-resident timing
        _barrier(ws)
        t0.record(stream)
        s_in.wait_event(t0)
        for i in range(e_steps):
            e2e_step(i)
        stream.wait_event(ev_out[0])
        stream.wait_event(ev_out[1])
        t1.record(stream)
        torch.cuda.synchronize()
        assert sage.sage_last_device_error() == 0
        ms_e2e = _max_over_ranks(t0.elapsed_time(t1) / e_steps, ws)
        # The same host->device copies alone (the step's input bytes over the
        # link, nothing else): the time the pipelined step cannot go below.
        qb, kb, vb, _ = bufs[0]
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        c0.record(s_in)
        with torch.cuda.stream(s_in):
            for _ in range(e_steps):
                qb.copy_(qh, non_blocking=True)
                kb.copy_(kh, non_blocking=True)
                vb.copy_(vh, non_blocking=True)
        c1.record(s_in)
        torch.cuda.synchronize()
        ms_h2d = _max_over_ranks(c0.elapsed_time(c1) / e_steps, ws)
        h2d_bytes = 3 * q.numel() * q.element_size()
        res["e2e"] = {"ms_step": ms_e2e, "h2d_bytes_per_step": h2d_bytes,
                      "d2h_bytes_per_step": o.numel() * o.element_size(), "steps": e_steps,
                      "pipelined": "double-buffered: copies of step i overlap the attention of step i-1",
                      "h2d_copy_ms": ms_h2d, "h2d_gbs": h2d_bytes / (ms_h2d * 1e-3) / 1e9}
        del bufs, ohs
    del wsp, qd, kd, vd, o
    torch.cuda.empty_cache()
    return res


# (kind, N) shapes of the tensor-core rate probe: M = 128 throughout; the
# attention kernels use i8 N = 128 (Q K^T), f8 N = d (P V) and f4 N = 128
MMA_SHAPES = (("i8", 256), ("i8", 128), ("i8", 64), ("f8", 256), ("f8", 128), ("f8", 64), ("f4", 128))


def measure_mma_peaks(target_ms: float = 30.0):
    """Measured tensor-core peaks of this GPU at the clocks of this run: the
    library's rate probe (one CTA per SM, back-to-back tcgen05.mma on resident
    shared-memory tiles) per kind and N, timed with CUDA events on the
    launching stream; each launch is sized to about target_ms."""
    from quantized_attention_block_b200 import sage

    stream = torch.cuda.current_stream()
    rates = {}
    with ClockSampler(torch.cuda.current_device()) as clk:
        clk.mark("timed", True)
        for kind, n in MMA_SHAPES:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            iters = 2000
            for _ in range(2):  # calibrate the length, then measure
                e0.record(stream)
                ops = sage.sage_debug_mma_rate(kind, n, iters, 0, stream)
                e1.record(stream)
                torch.cuda.synchronize()
                ms = e0.elapsed_time(e1)
                tops = ops / (ms * 1e-3) / 1e12
                iters = int(min(2_000_000, max(2000, iters * target_ms / max(ms, 1e-3))))
            rates[f"{kind}_n{n}"] = tops
        clk.mark("timed", False)
    assert sage.sage_last_device_error() == 0
    best = {k: max(v for key, v in rates.items() if key.startswith(k + "_")) for k in ("i8", "f8", "f4")}
    return {"tops": rates, "best": best, "clocks": clk.summary(),
            "how": "sage_debug_mma_rate: 1 CTA per SM, tcgen05.mma M=128 back to back on resident smem tiles, "
                   "CUDA events, ~%.0f ms per launch" % target_ms}


def oracle_sample(w: W.Workload, heads: int, tiles: int, threads: int, batches: int = 1):
    """Time the CPU oracle on a bounded sample: quantise `batches` x `heads`
    (b, h) pairs and run the attention of the last `tiles` Q tiles of each (the
    longest rows when causal).  Returns (seconds, attention ops, description)."""
    import numpy as np

    import oracle
    from concurrent.futures import ThreadPoolExecutor

    G = w.Hq // w.Hkv
    sw = w.with_(B=batches, Hq=heads * G if w.Hq != w.Hkv else heads, Hkv=heads if w.Hq != w.Hkv else heads)
    q, k, v = W.make_qkv(sw)
    n_t = -(-w.N // 128)
    jobs = [(b, h, t * 128, min((t + 1) * 128, w.N)) for b in range(batches) for h in range(sw.Hq)
            for t in range(n_t - tiles, n_t)]
    ops = 0.0
    for _, _, r0, r1 in jobs:
        for r in range(r0, r1):
            keys = (r + 1) if w.causal else w.N
            ops += 4.0 * keys * w.d
    t_start = time.perf_counter()
    quant = oracle.quantize_sage(q, k, v, bq=w.bq, bk=w.bk, smooth_k=w.smooth_k, smooth_q=w.smooth_q,
                                 threads=threads)
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(lambda j: oracle.attention_sage_head(quant, j[0], j[1], j[2], j[3], bq=w.bq, bk=w.bk,
                                                        causal=w.causal, sm_scale=w.sm_scale), jobs))
    secs = time.perf_counter() - t_start
    desc = (f"{batches} x {sw.Hq} heads of {w.name} (N={w.N}): full oracle quantisation of those heads + "
            f"attention of the last {tiles} Q tiles of each ({len(jobs)} tiles), {threads} threads")
    return secs, ops, desc


def main():
    faulthandler.enable()
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["sage", "reference"], default="sage")
    ap.add_argument("--workload", default="prefill")
    ap.add_argument("--extra-workloads", default="video,gqa,nvfp4")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--override", default="", help="workload fields, e.g. B=1,Hq=16,Hkv=16 (profiling cases)")
    ap.add_argument("--pv-accum", choices=["auto", "two_level", "tmem_fp32"], default="auto")
    ap.add_argument("--no-mma-peaks", action="store_true",
                    help="skip the tensor-core rate probe (the roofline then uses bf16 burst x nominal ratio)")
    args = ap.parse_args()

    ws, rank, local = _dist()
    w = W.get(args.workload)
    if args.override:
        kv = dict(x.split("=") for x in args.override.split(","))
        w = w.with_(name=w.name + "@" + args.override.replace(",", "_"), **{k: int(v) for k, v in kv.items()})
    metric = "quantized attn fwd TOPS on 1 B200 (N=4K-32K, d=64/128); % of tensor peak"
    threads = os.cpu_count() or 1
    config = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
              "causal": w.causal, "smooth_q": w.smooth_q, "bq": w.bq, "bk": w.bk,
              "input_dtype": str(w.dtype).replace("torch.", ""), "parallelism": f"replicas x{ws} (weak)",
              "l2": "inputs larger than L2 (Q/K/V bf16 and their quantised copies each exceed 126 MB)"}

    if args.impl == "reference":
        if rank != 0:
            return
        heads, tiles = (4, 2) if w.N >= 8192 else (8, 4)
        vals = []
        desc = ""
        if args.warmup > 0:
            oracle_sample(w, 1, 1, threads)
        for _ in range(args.steps):
            secs, ops, desc = oracle_sample(w, heads, tiles, threads)
            vals.append(ops / secs / 1e12)
        val = statistics.median(vals)
        print(json.dumps({
            "impl": "reference", "metric": metric, "value": val, "unit": "TOPS", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64 (int8/e4m3 codes, fp32 state)", "data": "synthetic",
            "config": config,
            "cpu_baseline": {"value": val, "unit": "TOPS", "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": val, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return

    if ws > 1:
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", device_id=torch.device("cuda", local),
                                             timeout=__import__("datetime").timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)

    peaks, peak_kind = _peaks()
    mode = pv_mode(w, args.pv_accum)
    config["pv_accum"] = ["two_level", "tmem_fp32"][mode]
    res = run_sage(w, args.steps, args.warmup, ws, rank, local, not args.no_e2e, mode,
                   time_other_mode=not args.no_e2e)
    ops = w.ops()
    value = weak_scaling_tops(ops, res["ms_step"], ws)
    attn_tops = ops / (res["ms_attn"] * 1e-3) / 1e12
    # roofline denominators: the tensor-core peaks measured in this run (the
    # INT8/FP8 kernel does equal Q K^T (i8) and P V (f8) work, so its peak is
    # the harmonic mean of the two rates); without the probe, bf16 burst x the
    # nominal dense ratio
    mma = None if args.no_mma_peaks else measure_mma_peaks()
    if mma is not None:
        b = mma["best"]
        peak_i8f8 = 2.0 / (1.0 / b["i8"] + 1.0 / b["f8"])
        peak_f4 = b["f4"]
        peak_src = (f"measured in this run (sage_debug_mma_rate): i8 {b['i8']:.0f}, f8 {b['f8']:.0f} TOPS "
                    f"(best N), harmonic mean for equal QK^T / PV work")
        peak_src_f4 = f"measured in this run (sage_debug_mma_rate): f4 {b['f4']:.0f} TOPS"
    else:
        peak_i8f8 = peaks["bf16_tflops"] * INT8_FP8_PER_BF16
        peak_f4 = peaks["bf16_tflops"] * FP4_PER_BF16
        peak_src = (f"{peak_kind}: bf16 burst {peaks['bf16_tflops']} x {INT8_FP8_PER_BF16} "
                    f"(nominal int8/fp8 : bf16)")
        peak_src_f4 = f"{peak_kind}: bf16 burst {peaks['bf16_tflops']} x {FP4_PER_BF16} (nominal fp4 : bf16)"
    peak_tops = peak_i8f8
    extra = {}
    for name in [x for x in args.extra_workloads.split(",") if x and x != "none"]:
        we = W.get(name)
        me = pv_mode(we, args.pv_accum)
        r = run_sage(we, max(3, args.steps // 4), 3, ws, rank, local, False, me, time_other_mode=True)
        pk = peak_f4 if we.nvfp4 else peak_i8f8
        extra[we.name] = {"pv_accum": "scaled_tmem_fp32" if we.nvfp4 else ["two_level", "tmem_fp32"][me],
                          "path": "nvfp4" if we.nvfp4 else "int8_fp8",
                          "step_tops": we.ops() / (r["ms_step"] * 1e-3) / 1e12,
                          "attn_kernel_tops": we.ops() / (r["ms_attn"] * 1e-3) / 1e12,
                          "ms_step": r["ms_step"], "ms_attn": r["ms_attn"],
                          "attn_frac_of_peak": we.ops() / (r["ms_attn"] * 1e-3) / 1e12 / pk,
                          "peak_tops": pk, "clocks": r["clocks"]}
        if "ms_attn_other_mode" in r:
            extra[we.name]["attn_kernel_tops_other_mode"] = we.ops() / (r["ms_attn_other_mode"] * 1e-3) / 1e12
            extra[we.name]["attn_frac_of_peak_other_mode"] = extra[we.name]["attn_kernel_tops_other_mode"] / pk
    line = {
        "metric": metric, "value": value, "unit": "TOPS", "n_gpus": ws, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": res["ms_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8+e4m3 (fp32 accumulate)",
        "data": "synthetic (seeded, recipe of the workload)", "config": config,
        "kernel_only_tops": attn_tops,
        "per_kernel_ms": {"quant_total": res["ms_quant"], "attn_i8f8": res["ms_attn"]},
        "attn_kernel_tops_other_pv_accum": (ops / (res["ms_attn_other_mode"] * 1e-3) / 1e12
                                            if "ms_attn_other_mode" in res else None),
        "roofline": {"bound": "tensor", "kernel": "attn_i8f8_kernel", "achieved": attn_tops,
                     "peak": peak_tops, "unit": "TFLOP/s", "frac": attn_tops / peak_tops,
                     "peak_source": peak_src, "peak_source_fp4": peak_src_f4,
                     "peak_bf16_burst_x_ratio": peaks["bf16_tflops"] * INT8_FP8_PER_BF16,
                     "traffic": _attn_traffic(w), "traffic_unit": "bytes per launch"},
        "clocks": res["clocks"], "gpu_launches": res["gpu_launches"], "workloads": extra,
    }
    if mma is not None:
        line["tensor_peaks_measured"] = mma
    if "e2e" in res:
        e = res["e2e"]
        line["e2e"] = {"value": weak_scaling_tops(ops, e["ms_step"], ws), "unit": "TOPS",
                       "h2d_bytes_per_step": e["h2d_bytes_per_step"], "d2h_bytes_per_step": e["d2h_bytes_per_step"],
                       "ms_step": e["ms_step"], "pipelined": e["pipelined"],
                       # the input copies alone over the host link: the bound of the pipelined step
                       "h2d_copy_ms_per_step": e["h2d_copy_ms"], "h2d_gbs": e["h2d_gbs"],
                       "copy_bound_frac": e["h2d_copy_ms"] / e["ms_step"]}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        # about 10-15 s on a 16-core host: three batches' worth of heads, the 32
        # longest Q tiles of each
        secs, ops_s, desc = oracle_sample(w, min(32, w.Hkv), 32, threads, batches=min(3, w.B))
        line["cpu_baseline"] = {"value": ops_s / secs / 1e12, "unit": "TOPS", "cores": threads, "kind": "oracle",
                                "sample": desc, "seconds": secs}
    if rank == 0:
        print(json.dumps(line))
    if ws > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

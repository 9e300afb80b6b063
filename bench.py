"""Benchmark: exact attention forward (long causal prefill) + paged-KV decode on B200.

One step is one pass of the whole hot path over one batch of synthetic input:
  1. attn_fwd on prefill_causal_b1_h16_l8192_d128_bf16 (tcgen05 prefill kernel), and
  2. attn_fwd_paged on paged_decode_s16_hq12_hkv2_d128_bf16 (paged decode kernel).
``value`` is the prefill's forward TFLOP/s (4*B*H*Lq*Lk*D, halved for causal) over the
prefill kernel's device time; the decode's HBM GB/s is reported beside it. Both kernels
are timed with CUDA events on the stream they run on. Inputs rotate over enough copies
that every step reads data that is not in L2.

After the step's timed region, two more calls on the same prefill workload are timed on
their own and reported beside ``value`` (not part of it): the backward pass (attn_bwd,
the ``backward`` object; --no-backward skips it) and the same prefill with K/V read
through a paged cache (attn_fwd_paged_prefill, the ``paged_prefill`` object;
--no-paged-prefill skips it), and the same prefill on e4m3 inputs (attn_fwd_fp8, the
``fp8`` object; --no-fp8 skips it).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 (launched by torch.distributed.run) every rank runs the same step on its own
GPU with its own inputs: independent problems, no collective on the data path (weak
scaling); rank 0 prints the whole-job throughput over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from tiled_attention_19_b200 import inputs  # noqa: E402

PREFILL = inputs.WORKLOADS["prefill_causal_b1_h16_l8192_d128_bf16"]
PREFILL_DEFAULT = PREFILL.name
DECODE = inputs.WORKLOADS["paged_decode_s16_hq12_hkv2_d128_bf16"]
METRIC = "fwd attention TFLOP/s & % of FP16 tensor peak; paged decode HBM GB/s"
L2_BYTES = 126 * 1000 * 1000
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Device code of each kernel the committed ncu traffic figures were taken on.
KERNEL_SOURCES = {
    name: ["tiled_attention_19_b200/csrc/" + f for f in ("common.cuh", "ptx.cuh", header)]
    for name, header in (("prefill", "prefill_sm100.cuh"), ("decode", "paged_decode.cuh"))
}


# ------------------------------------------------------------------------ helpers
def _find_number(d, key, depth=2):
    """d[key] as a float, looked up at the top level or up to `depth` levels of nested
    objects below it; None if absent or not a number."""
    if isinstance(d, dict):
        v = d.get(key)
        if isinstance(v, (int, float)) and not isinstance(v, bool) and v > 0:
            return float(v)
        if depth > 0:
            for sub in d.values():
                r = _find_number(sub, key, depth - 1)
                if r is not None:
                    return r
    return None


def load_peaks(path=None):
    """The measured peaks (hbm_gbs, bf16_tflops, bf16_tflops_sustained) from
    MEASURED_PEAKS.json; a key the file lacks (or a missing or unreadable file) takes the
    fallback figure, and the returned label says which."""
    p = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    d = None
    if os.path.exists(p):
        try:
            with open(p) as f:
                d = json.load(f)
        except (OSError, ValueError):
            d = None
    if d is None:
        return dict(PEAKS_FALLBACK), "fallback"
    peaks, missing = {}, []
    for k, fb in PEAKS_FALLBACK.items():
        v = _find_number(d, k)
        if v is None:
            missing.append(k)
            v = fb
        peaks[k] = v
    if not missing:
        return peaks, "measured"
    if len(missing) == len(PEAKS_FALLBACK):
        return peaks, "fallback"
    return peaks, "measured (fallback for " + ", ".join(missing) + ")"


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu summary,
    if it was taken on that kernel's device code as it is now (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get("kernels", {}).get(kernel, {})
    if e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("per_launch", {}).get(workload)


class ClockSampler:
    """SM clocks, power and clock-event (throttle) reasons, polled through NVML every
    few milliseconds from a background thread for the whole measurement, each sample
    stamped with the host clock; summary() keeps the samples inside a host-time window
    (the timed region), so even a region of a few milliseconds gets samples. Falls back
    to `nvidia-smi -lms` (50 ms period) where NVML cannot be loaded. Reads only."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    SMI_Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device, period_ms: float = 2.0):
        self.device, self.period = device, period_ms / 1e3
        self.samples = []  # (host time, sm MHz, max sm MHz, power W, [reasons])
        self.stop = threading.Event()
        self.thread = None
        self.proc = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
            except pynvml.NVMLError:
                pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = self.device.index or 0
        if vis:
            idx = int(vis.split(",")[idx])
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(idx)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            masks = [(n, getattr(nv, c)) for n, c in self.REASONS]
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)

            def poll():
                while not self.stop.is_set():
                    t = time.perf_counter()
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        pw = nv.nvmlDeviceGetPowerUsage(h) / 1e3
                        r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    except nv.NVMLError:
                        break
                    self.samples.append((t, float(sm), float(mx), pw,
                                         [n for n, m in masks if r & m]))
                    time.sleep(self.period)

            self.source = f"NVML, every {self.period * 1e3:.0f} ms"
        except Exception:  # no NVML: nvidia-smi at its shortest period
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.device.index or 0}", f"--query-gpu={self.SMI_Q}",
                     "--format=csv,noheader,nounits", "-lms=50"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except (OSError, ValueError):
                return self
            names = [n for n, _ in self.REASONS]

            def poll():
                for line in self.proc.stdout:
                    p = [x.strip() for x in line.split(",")]
                    if len(p) >= 9 and p[1].replace(".", "").isdigit():
                        self.samples.append((time.perf_counter(), float(p[1]), float(p[2]),
                                             float(p[3]) if p[3].replace(".", "").isdigit() else None,
                                             [n for n, v in zip(names, p[5:9]) if v == "Active"]))

            self.source = "nvidia-smi -lms 50"
        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()
        t0 = time.perf_counter()  # start measuring once the sampler delivers
        while not self.samples and time.perf_counter() - t0 < 5.0:
            time.sleep(0.005)
        return self

    def __exit__(self, *exc):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t_from: float, t_to: float):
        """Samples taken between host times t_from and t_to; if none fell inside (a
        region shorter than the period), the nearest sample on each side."""
        inside = [x for x in self.samples if t_from <= x[0] <= t_to]
        how = "inside the timed region"
        if not inside and self.samples:
            before = [x for x in self.samples if x[0] < t_from][-1:]
            after = [x for x in self.samples if x[0] > t_to][:1]
            inside = before + after
            how = "nearest samples on either side of the timed region"
        if not inside:
            return None
        sm = [x[1] for x in inside]
        pw = [x[3] for x in inside if x[3] is not None]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(x[2] for x in inside),
                "sm_min_mhz": min(sm), "power_w": round(statistics.median(pw), 1) if pw else None,
                "reasons": sorted({r for x in inside for r in x[4]}), "samples": len(inside),
                "source": f"{self.source}; {how}"}


DENSE_BF16_FLOP_PER_CLOCK_PER_SM = 8192  # 2.25 PFLOP/s dense at about 1.855 GHz on 148 SMs


def clock_peak_fields(tflops, clock_record, device) -> dict:
    """The nominal dense bf16 tensor rate at the SM clock actually seen in the timed
    region (SMs x 8192 FLOP per clock x the median SM clock) and the fraction of it, so
    that a power-capped or throttled run reads against the rate it ran at."""
    mhz = (clock_record or {}).get("sm_mhz")
    if not tflops or not mhz:
        return {"clock_peak": None, "frac_of_clock_peak": None}
    try:
        sms = torch.cuda.get_device_properties(device).multi_processor_count
    except (RuntimeError, AssertionError, AttributeError):
        return {"clock_peak": None, "frac_of_clock_peak": None}
    peak = sms * DENSE_BF16_FLOP_PER_CLOCK_PER_SM * float(mhz) * 1e6 / 1e12
    return {"clock_peak": round(peak, 1), "frac_of_clock_peak": round(tflops / peak, 4),
            "clock_peak_note": f"{sms} SMs x {DENSE_BF16_FLOP_PER_CLOCK_PER_SM} dense bf16 FLOP per "
                               f"clock x the median SM clock in the timed region ({mhz:.0f} MHz)"}


def tensor_peak(peaks: dict, region_ms: float):
    """The measured tensor peak that applies to a kernel timed over `region_ms`: the
    burst GEMM rate below one second of timed work, the sustained (power-capped) rate
    above it."""
    if region_ms < 1000.0:
        return peaks["bf16_tflops"], "bf16_tflops (burst: the timed region is under 1 s)"
    return peaks["bf16_tflops_sustained"], "bf16_tflops_sustained (the timed region is over 1 s)"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(x: float, ws: int, device) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def job_rate(work_per_rank: float, ms_max_over_ranks: float, ws: int, unit_scale: float):
    """Whole-job throughput of weak-scaled replicas: every rank processes the same
    amount of work, and the job takes as long as the slowest rank."""
    if not (ms_max_over_ranks == ms_max_over_ranks) or ms_max_over_ranks <= 0:
        return None
    return ws * work_per_rank / (ms_max_over_ranks * 1e-3) / unit_scale


# ----------------------------------------------------------------- our GPU arm
class Workload:
    """Device copies of the step's inputs (rotated) and its outputs."""

    def __init__(self, device, copies: int, window=None):
        self.device = device
        xp = inputs.make(PREFILL)
        xd = inputs.make(DECODE)
        self.xp_host, self.xd_host = xp, xd
        # enough prefill copies that one rotation spans more than twice the 126 MB L2
        per_copy = sum(v.numel() * v.element_size() for v in xp.values())
        self.p_copies = max(copies, -(-2 * L2_BYTES // per_copy)) if copies > 1 else 1
        self.pf = [{k: v.to(device) for k, v in xp.items()} for _ in range(self.p_copies)]
        # and enough decode copies that the bytes one rotation's calls touch (the valid
        # tokens' K/V rows, not the whole pool) also span more than twice the L2
        self.decode_bytes = inputs.paged_bytes(DECODE, xd["seq_lens"])
        self.d_copies = max(copies, -(-2 * L2_BYTES // self.decode_bytes)) if copies > 1 else 1
        self.dc = [{k: v.to(device) for k, v in xd.items()} for _ in range(self.d_copies)]
        self.copies = copies
        self.p_out = torch.empty_like(self.pf[0]["q"])
        self.p_lse = torch.empty(PREFILL.B, PREFILL.Hq, PREFILL.Lq, device=device)
        self.prefill_bytes = inputs.dense_bytes(PREFILL)
        self.d_out = torch.empty_like(self.dc[0]["q"])
        self.d_lse = torch.empty(DECODE.num_seqs, DECODE.Hq, device=device)
        self.prefill_flops = PREFILL.flops() if window is None else windowed_flops(PREFILL, window)


def windowed_flops(spec, window) -> float:
    """4 * D FLOPs per visible (query row, key) pair, counted exactly for a band:
    row i (i' = i + Lk - Lq) sees keys max(0, i'-left) .. min(Lk-1, i'+right)."""
    left, right = window
    if spec.causal:
        right = 0
    i = torch.arange(spec.Lq, dtype=torch.int64) + (spec.Lk - spec.Lq)
    lo = torch.clamp(i - left, min=0) if left >= 0 else torch.zeros_like(i)
    hi = torch.clamp(i + right, max=spec.Lk - 1) if right >= 0 else torch.full_like(i, spec.Lk - 1)
    pairs = int(torch.clamp(hi - lo + 1, min=0).sum())
    return 4.0 * spec.D * spec.B * spec.Hq * pairs


SMALL_CONFIGS = ("sdpa_b1_h8_l512_d64_f16", "vit_b32_h12_n196_d64_f16",
                 "sdpa_causal_b2_h8_l2048_d64_f16")


def run_ours(args, ws, rank, local):
    import tiled_attention_19_b200 as ta
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    ta.load()
    clocks = ClockSampler(device)
    clocks.__enter__()  # samples the whole run; each timed region picks its own window
    try:
        return _run_ours(args, ws, rank, ta, device, clocks)
    finally:
        clocks.__exit__(None, None, None)


def _run_ours(args, ws, rank, ta, device, clocks):
    copies = args.copies  # at least this many copies of each input (more where L2 needs it)
    w = Workload(device, copies, args.window)
    do_pre = args.only in ("both", "prefill")
    do_dec = args.only in ("both", "decode")
    stream = torch.cuda.current_stream()
    ws_buf = ta.paged_workspace(DECODE.num_seqs, DECODE.Hq, DECODE.Hkv, DECODE.D,
                                DECODE.max_blocks, device)

    def step(i, ev=None):
        p = w.pf[i % w.p_copies]
        d = w.dc[i % w.d_copies]
        if ev is not None:
            ev[0].record(stream)
        if do_pre:
            ta.fwd(p["q"], p["k"], p["v"], causal=PREFILL.causal, scale=PREFILL.scale, out=w.p_out,
                   lse=w.p_lse, stream=stream, window=args.window)
        if ev is not None:
            ev[1].record(stream)
        if do_dec:
            ta.fwd_paged(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["seq_lens"],
                         scale=DECODE.scale, out=w.d_out, lse=w.d_lse, workspace=ws_buf,
                         stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    status = ta.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    h0 = time.perf_counter()
    t0.record(stream)
    for i in range(args.steps):
        step(args.warmup + i, evs[i])
    host_ms = (time.perf_counter() - h0) * 1e3  # host time to enqueue the K steps
    t1.record(stream)
    torch.cuda.synchronize()
    h1 = time.perf_counter()
    barrier(ws)
    region_clocks = clocks.summary(h0, h1)
    total_ms = t0.elapsed_time(t1)
    pre_ms = [e[0].elapsed_time(e[1]) for e in evs]
    dec_ms = [e[1].elapsed_time(e[2]) for e in evs]
    if ta.device_status() != 0:
        raise RuntimeError("device status set during the timed region")

    total_ms = reduce_max(total_ms, ws, device)
    pre_avg = reduce_max(sum(pre_ms) / len(pre_ms), ws, device)
    dec_avg = reduce_max(sum(dec_ms) / len(dec_ms), ws, device)

    # The same calls replayed from CUDA graphs: device time per launch without the
    # host's launch latency (matters for microsecond kernels such as the decode).
    g_pre = g_dec = None
    if args.graphs:
        if do_pre:
            g_pre = graph_launch_ms(
                lambda i: ta.fwd(w.pf[i % w.p_copies]["q"], w.pf[i % w.p_copies]["k"],
                                 w.pf[i % w.p_copies]["v"], causal=PREFILL.causal,
                                 scale=PREFILL.scale, out=w.p_out, lse=w.p_lse,
                                 window=args.window),
                n_calls=2 * w.p_copies, replays=max(1, min(100, args.steps) // (2 * w.p_copies)),
                ws=ws, device=device)
        if do_dec:
            g_dec = graph_launch_ms(
                lambda i: ta.fwd_paged(w.dc[i % w.d_copies]["q"], w.dc[i % w.d_copies]["k_cache"],
                                       w.dc[i % w.d_copies]["v_cache"], w.dc[i % w.d_copies]["block_table"],
                                       w.dc[i % w.d_copies]["seq_lens"], scale=DECODE.scale,
                                       out=w.d_out, lse=w.d_lse, workspace=ws_buf),
                n_calls=2 * w.d_copies, replays=max(1, min(1000, args.steps) // (2 * w.d_copies)),
                ws=ws, device=device)

    cfg = None
    if args.configs and args.window is None:
        cfg = measure_configs(ta, device, ws, steps=max(20, min(200, args.steps)),
                              warmup=args.warmup, clocks=clocks)

    bwd_ms = None
    if args.backward and do_pre:
        bwd_ms = measure_backward(w, ta, stream, device, steps=max(3, min(100, args.steps)),
                                  warmup=args.warmup, ws=ws, window=args.window)

    pp_ms = None
    if args.paged_prefill and do_pre and args.window is None and PREFILL.Lq == PREFILL.Lk \
            and PREFILL.Lk % 16 == 0:
        pp_ms = measure_paged_prefill(w, ta, stream, device, steps=max(3, min(300, args.steps)),
                                      warmup=args.warmup, ws=ws)

    fp8_ms = None
    if args.fp8 and do_pre and args.window is None and PREFILL.D == 128:
        fp8_ms = measure_fp8(w, ta, stream, device, steps=max(3, min(300, args.steps)),
                             warmup=args.warmup, ws=ws)

    if args.e2e:
        e2e = measure_e2e(w, ta, stream, device, steps=max(3, min(20, args.steps)), window=args.window)
    else:
        e2e = {"prefill_ms": float("nan"), "decode_ms": float("nan"), "h2d_bytes": 0,
               "d2h_bytes": 0, "serial_prefill_ms": float("nan"), "serial_decode_ms": float("nan")}
    e2e_pre = reduce_max(e2e["prefill_ms"], ws, device)
    e2e_dec = reduce_max(e2e["decode_ms"], ws, device)
    e2e_pre_serial = reduce_max(e2e["serial_prefill_ms"], ws, device)
    e2e_dec_serial = reduce_max(e2e["serial_decode_ms"], ws, device)

    if rank != 0:
        return None
    peaks, peaks_src = load_peaks()

    tflops = job_rate(w.prefill_flops, pre_avg, ws, 1e12) if do_pre else None
    gbs = job_rate(w.decode_bytes, dec_avg, ws, 1e9) if do_dec else None
    per_gpu_tflops = tflops / ws if tflops is not None else None
    per_gpu_gbs = gbs / ws if gbs is not None else None
    r2 = lambda x, n: None if x is None else round(x, n)  # noqa: E731
    e2e_tf = job_rate(w.prefill_flops, e2e_pre, ws, 1e12) if do_pre else None
    e2e_gb = job_rate(w.decode_bytes, e2e_dec, ws, 1e9) if do_dec else None
    e2e_tf_serial = job_rate(w.prefill_flops, e2e_pre_serial, ws, 1e12) if do_pre else None
    e2e_gb_serial = job_rate(w.decode_bytes, e2e_dec_serial, ws, 1e9) if do_dec else None
    pk_t, pk_t_src = tensor_peak(peaks, total_ms)
    pk_h = peaks["hbm_gbs"]
    line = {
        "metric": METRIC,
        "value": r2(tflops, 2),
        "unit": "TFLOP/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4),
        "host_ms_per_step": round(host_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) inputs shaped like the pages' workloads)",
        "config": {
            "workload": f"{PREFILL.name} + {DECODE.name}",
            "prefill": {"B": PREFILL.B, "H": PREFILL.Hq, "Lq": PREFILL.Lq, "Lk": PREFILL.Lk,
                        "D": PREFILL.D, "causal": PREFILL.causal,
                        "dtype": "bf16" if PREFILL.dtype == torch.bfloat16 else "f16",
                        "flops": w.prefill_flops},
            "decode": {"seqs": DECODE.num_seqs, "Hq": DECODE.Hq, "Hkv": DECODE.Hkv,
                       "D": DECODE.D, "block_size": DECODE.block_size,
                       "tokens": int(w.xd_host["seq_lens"].sum()),
                       "bytes": w.decode_bytes},
            "l2": f"inputs rotate over device copies larger than the 126 MB L2: prefill "
                  f"{w.p_copies} x {sum(v.numel() * v.element_size() for v in w.xp_host.values()) / 1e6:.1f} MB, "
                  f"decode {w.d_copies} x {w.decode_bytes / 1e6:.1f} MB touched per call (pools of "
                  f"{sum(v.numel() * v.element_size() for v in w.xd_host.values()) / 1e6:.0f} MB)",
            "parallelism": f"replicas x{ws} (independent problems per GPU)",
            "window": args.window,
        },
        "roofline": {
            "kernel": f"prefill_fwd_kernel<{PREFILL.D},{'bf16' if PREFILL.dtype == torch.bfloat16 else 'f16'},"
                      f"{'causal' if PREFILL.causal else 'full'}>",
            "bound": "tensor",
            "achieved": r2(per_gpu_tflops, 2),
            "peak": pk_t,
            "peak_source": f"{peaks_src} {pk_t_src}",
            "unit": "TFLOP/s",
            "frac": r2(per_gpu_tflops and per_gpu_tflops / pk_t, 4),
            "frac_of_sustained_peak": r2(per_gpu_tflops and per_gpu_tflops / peaks["bf16_tflops_sustained"], 4),
            **clock_peak_fields(per_gpu_tflops, region_clocks, device),
            "traffic": None if args.window else profiled_traffic("prefill", PREFILL.name),
            "timed_region_ms": round(total_ms, 3),
            "avg_launch_ms": round(pre_avg, 5),
            "graph_avg_launch_ms": None if g_pre is None else round(g_pre, 5),
            "graph_frac": None if g_pre is None else r2(w.prefill_flops / (g_pre * 1e-3) / 1e12 / pk_t, 4),
        },
        "paged_decode": {
            "kernel": "paged_decode_kernel<128,bf16>",
            "value": r2(gbs, 1),
            "unit": "GB/s",
            "bound": "hbm",
            "achieved": r2(per_gpu_gbs, 1),
            "peak": pk_h,
            "peak_source": f"{peaks_src} hbm_gbs",
            "frac": r2(per_gpu_gbs and per_gpu_gbs / pk_h, 4),
            "traffic": profiled_traffic("decode", DECODE.name),
            "avg_launch_ms": round(dec_avg, 5),
            "graph_avg_launch_ms": None if g_dec is None else round(g_dec, 5),
            "graph_value": None if g_dec is None else r2(w.decode_bytes / (g_dec * 1e-3) / 1e9, 1),
            "graph_frac": None if g_dec is None else r2(w.decode_bytes / (g_dec * 1e-3) / 1e9 / pk_h, 4),
            "graph_note": "the same calls replayed back to back from a CUDA graph (no host work "
                          "between launches); avg_launch_ms above includes the host's launch "
                          "latency whenever it exceeds the kernel's time",
        },
        "e2e": {
            "value": r2(e2e_tf, 3),
            "unit": "TFLOP/s",
            "h2d_bytes_per_step": e2e["h2d_bytes"],
            "d2h_bytes_per_step": e2e["d2h_bytes"],
            "paged_decode_gbs": r2(e2e_gb, 2),
            "how": "every step copies its inputs from pinned host memory to the device, makes the "
                   "C-ABI call and copies its outputs back, all inside the timed region; two "
                   "buffer sets let step i+1's host-to-device copies overlap step i's call and "
                   "step i-1's device-to-host copies (three streams, event-ordered). The prefill "
                   "and the decode each run such a loop: value is the prefill's TFLOP/s over its "
                   "loop, paged_decode_gbs the decode's; the byte counts are one whole step's "
                   "(prefill and decode inputs and outputs)",
            "serial_value": r2(e2e_tf_serial, 3),
            "serial_paged_decode_gbs": r2(e2e_gb_serial, 2),
            "serial_how": "the same steps on one stream with a host sync after each step",
        },
        "gpu_launches": (int(do_pre) + int(do_dec)) * args.steps,
        "clocks": region_clocks,
    }
    if cfg is not None:
        line["configs"] = {}
        for name, c in cfg.items():
            spec = inputs.WORKLOADS[name]
            pk, pk_src = tensor_peak(peaks, c["region_ms"])
            tf = spec.flops() / (c["ms"] * 1e-3) / 1e12
            gtf = None if c["graph_ms"] is None else spec.flops() / (c["graph_ms"] * 1e-3) / 1e12
            nbytes = inputs.dense_bytes(spec)
            line["configs"][name] = {
                "kernel": f"prefill_fwd_kernel<{spec.D},{'bf16' if spec.dtype == torch.bfloat16 else 'f16'},"
                          f"{'causal' if spec.causal else 'full'}>",
                "flops": spec.flops(),
                "bytes": nbytes,
                "avg_launch_ms": round(c["ms"], 5),
                "value": r2(tf, 2),
                "unit": "TFLOP/s",
                "bound": "tensor",
                "peak": pk,
                "peak_source": f"{peaks_src} {pk_src}",
                "frac": r2(tf / pk, 4),
                "graph_avg_launch_ms": None if c["graph_ms"] is None else round(c["graph_ms"], 5),
                "graph_value": r2(gtf, 2),
                "graph_frac": None if gtf is None else r2(gtf / pk, 4),
                "graph_gbs": None if c["graph_ms"] is None else r2(nbytes / (c["graph_ms"] * 1e-3) / 1e9, 1),
                "graph_hbm_frac": None if c["graph_ms"] is None else
                r2(nbytes / (c["graph_ms"] * 1e-3) / 1e9 / pk_h, 4),
                "launches": c["launches"],
                "copies": c["copies"],
                "clocks": c["clocks"],
                "bar": "tensor >= 0.60 of peak (L >= 2048)" if spec.Lq >= 2048 else None,
            }
    if pp_ms is not None:
        pp_tf = job_rate(w.prefill_flops, pp_ms, ws, 1e12) / ws
        pk_pp, pk_pp_src = tensor_peak(peaks, pp_ms * max(3, min(300, args.steps)))
        line["paged_prefill"] = {
            "what": "attn_fwd_paged_prefill on the prefill workload with K/V scattered over a "
                    "paged cache (16-token blocks, seeded permutation), the whole sequence as "
                    "the chunk",
            "kernel": f"prefill_fwd_kernel<{PREFILL.D},paged>",
            "value": r2(pp_tf * ws, 2),
            "unit": "TFLOP/s",
            "bound": "tensor",
            "achieved": r2(pp_tf, 2),
            "peak": pk_pp,
            "peak_source": f"{peaks_src} {pk_pp_src}",
            "frac": r2(pp_tf / pk_pp, 4),
            "vs_dense": r2(pre_avg / pp_ms, 4),
            "avg_call_ms": round(pp_ms, 5),
            "steps": max(3, min(300, args.steps)),
            "gpu_launches": max(3, min(300, args.steps)),
        }
    if fp8_ms is not None:
        f8_tf = job_rate(w.prefill_flops, fp8_ms, ws, 1e12) / ws
        pk_b, pk_b_src = tensor_peak(peaks, fp8_ms * max(3, min(300, args.steps)))
        pk_f8 = 2 * pk_b  # the fp8 tensor rate is twice the bf16 rate (nominal 4.5 vs 2.25 PFLOP/s)
        line["fp8"] = {
            "what": "attn_fwd_fp8 on the prefill workload with q, k, v cast to e4m3 (bf16 output)",
            "kernel": f"prefill_fwd_kernel<{PREFILL.D},e4m3>",
            "value": r2(f8_tf * ws, 2),
            "unit": "TFLOP/s",
            "bound": "tensor",
            "achieved": r2(f8_tf, 2),
            "peak": pk_f8,
            "peak_source": f"{peaks_src} {pk_b_src} x 2 (nominal fp8/bf16 ratio)",
            "frac": r2(f8_tf / pk_f8, 4),
            "vs_bf16": r2(pre_avg / fp8_ms, 4),
            "avg_call_ms": round(fp8_ms, 5),
            "steps": max(3, min(300, args.steps)),
            "gpu_launches": max(3, min(300, args.steps)),
        }
    if bwd_ms is not None:
        bwd_flops = 2.5 * w.prefill_flops
        bwd_tf = job_rate(bwd_flops, bwd_ms, ws, 1e12) / ws
        pk_bw, pk_bw_src = tensor_peak(peaks, bwd_ms * max(3, min(100, args.steps)))
        line["backward"] = {
            "what": "attn_bwd of the prefill workload: dQ, dK, dV from O, lse and a seeded dO",
            "kernels": "bwd_prep_kernel + bwd_kernel<dK,dV> + bwd_kernel<dQ>",
            "value": r2(bwd_tf * ws, 2),
            "unit": "TFLOP/s",
            "flops": bwd_flops,
            "flops_note": "algorithmic: 2.5 x the forward's (five D-deep products per visible "
                          "pair); the kernels execute seven (S and dP are recomputed by both "
                          "the dK/dV and the dQ kernel), so 5/7 of the peak is their ceiling",
            "bound": "tensor",
            "achieved": r2(bwd_tf, 2),
            "peak": pk_bw,
            "peak_source": f"{peaks_src} {pk_bw_src}",
            "frac": r2(bwd_tf / pk_bw, 4),
            "avg_call_ms": round(bwd_ms, 5),
            "steps": max(3, min(100, args.steps)),
            "gpu_launches": 3 * max(3, min(100, args.steps)),
        }
    if args.cpu_baseline and ws == 1:
        gpu = {"prefill": (w.p_out, w.p_lse) if do_pre and args.window is None else None,
               "decode": (w.d_out, w.d_lse) if do_dec else None,
               "configs": {n: (c["inputs"], c["out"], c["lse"]) for n, c in (cfg or {}).items()}}
        line["cpu_baseline"], line["parity"] = cpu_baseline(args.cpu_seconds, gpu)
    return line


def measure_configs(ta, device, ws, steps: int, warmup: int, clocks):
    """The pages' smaller dense workloads (B1 H8 L512, the ViT-B/16 attention, B2 H8 L2048
    causal; fp16, D = 64), each timed on its own: `steps` back-to-back attn_fwd calls
    between two CUDA events, and the same calls replayed from a CUDA graph. Inputs rotate
    over device copies that together exceed twice the L2. Returns per workload the ms per
    launch, the graph's ms per launch, the clock record of the timed window and the
    output of one call (for the oracle comparison)."""
    res = {}
    stream = torch.cuda.current_stream()
    for name in SMALL_CONFIGS:
        spec = inputs.WORKLOADS[name]
        x = inputs.make(spec)
        per = sum(t.numel() * t.element_size() for t in x.values())
        n_copies = max(2, -(-2 * L2_BYTES // per))
        dev = [{k: v.to(device) for k, v in x.items()} for _ in range(n_copies)]
        out = torch.empty_like(dev[0]["q"])
        lse = torch.empty(spec.B, spec.Hq, spec.Lq, device=device)

        def call(i, st=None):
            c = dev[i % n_copies]
            ta.fwd(c["q"], c["k"], c["v"], causal=spec.causal, scale=spec.scale, out=out,
                   lse=lse, stream=st)

        for i in range(warmup):
            call(i, stream)
        torch.cuda.synchronize()
        if ta.device_status() != 0:
            raise RuntimeError(f"device status set by the {name} warm-up")
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(ws)
        torch.cuda.synchronize()
        h0 = time.perf_counter()
        e0.record(stream)
        for i in range(steps):
            call(warmup + i, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        h1 = time.perf_counter()
        barrier(ws)
        ms = reduce_max(e0.elapsed_time(e1) / steps, ws, device)
        n_calls = max(2 * n_copies, 64)
        g_ms = graph_launch_ms(lambda i: call(i), n_calls=n_calls,
                               replays=max(1, 2000 // n_calls), ws=ws, device=device)
        if ta.device_status() != 0:
            raise RuntimeError(f"device status set during the {name} timing")
        call(0, stream)
        torch.cuda.synchronize()
        res[name] = {"ms": ms, "graph_ms": g_ms, "region_ms": ms * steps, "launches": steps,
                     "copies": n_copies, "clocks": clocks.summary(h0, h1), "inputs": x,
                     "out": out, "lse": lse}
        del dev
    return res


def measure_backward(w, ta, stream, device, steps: int, warmup: int, ws: int, window=None):
    """The backward pass (attn_bwd) of the prefill workload, timed on its own after the
    step: dO is seeded like the inputs, O and lse come from one forward call per input
    copy, and the calls rotate over the copies as the step does."""
    do_host = inputs.dense_grad_output(PREFILL)
    sets = []
    for p in w.pf:
        out, lse = ta.fwd(p["q"], p["k"], p["v"], causal=PREFILL.causal, scale=PREFILL.scale,
                          window=window, stream=stream)
        sets.append((p, out, lse, do_host.to(device)))
    dq = torch.empty_like(w.pf[0]["q"])
    dk = torch.empty_like(w.pf[0]["k"])
    dv = torch.empty_like(w.pf[0]["v"])
    wsb = torch.empty(max(16, ta.bwd_workspace_size(PREFILL.B, PREFILL.Hq, PREFILL.Lq)),
                      dtype=torch.uint8, device=device)

    def call(i):
        p, out, lse, do = sets[i % len(sets)]
        ta.bwd(p["q"], p["k"], p["v"], out, do, lse, causal=PREFILL.causal, scale=PREFILL.scale,
               window=window, dq=dq, dk=dk, dv=dv, workspace=wsb, stream=stream)

    for i in range(warmup):
        call(i)
    torch.cuda.synchronize()
    if ta.device_status() != 0:
        raise RuntimeError("device status set by the backward warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    barrier(ws)
    torch.cuda.synchronize()
    for i in range(steps):
        ev[i][0].record(stream)
        call(warmup + i)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    if ta.device_status() != 0:
        raise RuntimeError("device status set during the backward timing")
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    return reduce_max(ms, ws, device)


def graph_launch_ms(call, n_calls: int, replays: int, ws: int, device):
    """Per-launch device time of `call` from a CUDA graph of n_calls back-to-back calls,
    replayed `replays` times between two events: no host work between launches, so a
    kernel of a few microseconds is timed without the host's launch latency. None if the
    capture fails."""
    try:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for i in range(3):
                call(i)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n_calls):
                call(i)
        g.replay()
        torch.cuda.synchronize()
    except RuntimeError:
        return None
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(replays):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    barrier(ws)
    ms = e0.elapsed_time(e1) / (replays * n_calls)
    del g
    return reduce_max(ms, ws, device)


def measure_paged_prefill(w, ta, stream, device, steps: int, warmup: int, ws: int):
    """The same prefill through a paged cache (attn_fwd_paged_prefill), timed on its own:
    each input copy's K and V are cut into 16-token blocks and scattered over the pool by
    one seeded permutation; the chunk is the whole sequence. Returns ms per call."""
    B, H, L, D = PREFILL.B, PREFILL.Hkv, PREFILL.Lk, PREFILL.D
    nblk = L // 16
    g = torch.Generator().manual_seed(PREFILL.seed + 17)
    perm = torch.randperm(B * nblk, generator=g).to(device)
    table = perm.view(B, nblk).to(torch.int32)
    seq_lens = torch.full((B,), L, dtype=torch.int32, device=device)
    sets = []
    for p in w.pf:
        caches = []
        for t in (p["k"], p["v"]):
            blocks = t.view(B, H, nblk, 16, D).permute(0, 2, 1, 3, 4).reshape(B * nblk, H, 16, D)
            c = torch.empty((B * nblk, H, 16, D), dtype=t.dtype, device=t.device)
            c[perm] = blocks
            caches.append(c)
        sets.append((p["q"], caches[0], caches[1]))
    out = torch.empty_like(w.pf[0]["q"])
    lse = torch.empty(B, PREFILL.Hq, PREFILL.Lq, device=device)

    def call(i):
        q, kc, vc = sets[i % len(sets)]
        ta.fwd_paged_prefill(q, kc, vc, table, seq_lens, causal=PREFILL.causal,
                             scale=PREFILL.scale, out=out, lse=lse, stream=stream)

    for i in range(warmup):
        call(i)
    torch.cuda.synchronize()
    if ta.device_status() != 0:
        raise RuntimeError("device status set by the paged-prefill warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    barrier(ws)
    torch.cuda.synchronize()
    for i in range(steps):
        ev[i][0].record(stream)
        call(warmup + i)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    if ta.device_status() != 0:
        raise RuntimeError("device status set during the paged-prefill timing")
    return reduce_max(sum(a.elapsed_time(b) for a, b in ev) / steps, ws, device)


def measure_fp8(w, ta, stream, device, steps: int, warmup: int, ws: int):
    """The same prefill on e4m3 inputs (attn_fwd_fp8), timed on its own: each input
    copy's q, k, v are cast to float8_e4m3fn once. Returns ms per call."""
    sets = [tuple(p[n].to(torch.float8_e4m3fn) for n in ("q", "k", "v")) for p in w.pf]
    out = torch.empty(PREFILL.B, PREFILL.Hq, PREFILL.Lq, PREFILL.D, dtype=torch.bfloat16,
                      device=device)
    lse = torch.empty(PREFILL.B, PREFILL.Hq, PREFILL.Lq, device=device)

    def call(i):
        q, k, v = sets[i % len(sets)]
        ta.fwd_fp8(q, k, v, causal=PREFILL.causal, scale=PREFILL.scale, out=out, lse=lse,
                   stream=stream)

    for i in range(warmup):
        call(i)
    torch.cuda.synchronize()
    if ta.device_status() != 0:
        raise RuntimeError("device status set by the fp8 warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    barrier(ws)
    torch.cuda.synchronize()
    for i in range(steps):
        ev[i][0].record(stream)
        call(warmup + i)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    if ta.device_status() != 0:
        raise RuntimeError("device status set during the fp8 timing")
    return reduce_max(sum(a.elapsed_time(b) for a, b in ev) / steps, ws, device)


def _pipelined_ms(host_in: dict, out_like: dict, call, steps: int, warmup: int, device) -> float:
    """ms per step of a double-buffered loop through the public API: the H2D copies of
    step i+1 (one copy stream) overlap the call of step i (a compute stream) and the D2H
    copies of step i-1 (a second copy stream). Every step's copies are inside the timed
    region, which runs from the first timed H2D to the last D2H."""
    sets = 2
    dev_in = [{k: torch.empty_like(v, device=device) for k, v in host_in.items()} for _ in range(sets)]
    dev_out = [{k: torch.empty_like(v, device=device) for k, v in out_like.items()} for _ in range(sets)]
    host_out = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in out_like.items()}
    s_in, s_run, s_out = (torch.cuda.Stream(device) for _ in range(3))
    n = warmup + steps
    ev_in = [torch.cuda.Event() for _ in range(n)]
    ev_run = [torch.cuda.Event() for _ in range(n)]
    ev_out = [torch.cuda.Event() for _ in range(n)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    for i in range(n):
        if i == warmup:  # the timed region starts once the warm-up steps have drained
            torch.cuda.synchronize()
            t0.record(s_in)
        b = i % sets
        if i >= sets:
            s_in.wait_event(ev_run[i - sets])   # step i-2's call read input set b
        with torch.cuda.stream(s_in):
            for k, v in host_in.items():
                dev_in[b][k].copy_(v, non_blocking=True)
        ev_in[i].record(s_in)
        s_run.wait_event(ev_in[i])
        if i >= sets:
            s_run.wait_event(ev_out[i - sets])  # step i-2's D2H read output set b
        call(dev_in[b], dev_out[b], s_run)
        ev_run[i].record(s_run)
        s_out.wait_event(ev_run[i])
        with torch.cuda.stream(s_out):
            for k, v in host_out.items():
                v.copy_(dev_out[b][k], non_blocking=True)
        ev_out[i].record(s_out)
    t1.record(s_out)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps


def measure_e2e(w, ta, stream, device, steps: int, window=None):
    """Same metric through the public API with host buffers: H2D of the step's inputs
    from pinned memory, the call, D2H of its outputs, all inside the timed region.
    Reported: a double-buffered loop (copies in both directions overlap the calls, as a
    serving loop would run them) and, for context, the same steps one after another on
    one stream with a host sync per step."""
    hp = {k: v.pin_memory() for k, v in w.xp_host.items()}
    hd = {k: v.pin_memory() for k, v in w.xd_host.items()}
    wsb = ta.paged_workspace(DECODE.num_seqs, DECODE.Hq, DECODE.Hkv, DECODE.D, DECODE.max_blocks,
                             device)
    p_like = {"out": w.p_out, "lse": w.p_lse}
    d_like = {"out": w.d_out, "lse": w.d_lse}
    h2d = sum(v.numel() * v.element_size() for v in list(hp.values()) + list(hd.values()))
    d2h = sum(t.numel() * t.element_size() for t in list(p_like.values()) + list(d_like.values()))

    def pre_call(di, do, st):
        ta.fwd(di["q"], di["k"], di["v"], causal=PREFILL.causal, scale=PREFILL.scale,
               out=do["out"], lse=do["lse"], stream=st, window=window)

    def dec_call(di, do, st):
        ta.fwd_paged(di["q"], di["k_cache"], di["v_cache"], di["block_table"], di["seq_lens"],
                     scale=DECODE.scale, out=do["out"], lse=do["lse"], workspace=wsb, stream=st)

    pre_ms = _pipelined_ms(hp, p_like, pre_call, steps, 2, device)
    dec_ms = _pipelined_ms(hd, d_like, dec_call, steps, 2, device)

    # the serial form: one stream, H2D -> call -> D2H, a host sync after every step
    dp = {k: torch.empty_like(v, device=device) for k, v in hp.items()}
    dd = {k: torch.empty_like(v, device=device) for k, v in hd.items()}
    op = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in p_like.items()}
    od = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in d_like.items()}
    pre, dec = [], []
    for it in range(steps + 1):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        with torch.cuda.stream(stream):
            for k in dp:
                dp[k].copy_(hp[k], non_blocking=True)
            pre_call(dp, p_like, stream)
            for k in op:
                op[k].copy_(p_like[k], non_blocking=True)
        e[1].record(stream)
        with torch.cuda.stream(stream):
            for k in dd:
                dd[k].copy_(hd[k], non_blocking=True)
            dec_call(dd, d_like, stream)
            for k in od:
                od[k].copy_(d_like[k], non_blocking=True)
        e[2].record(stream)
        torch.cuda.synchronize()
        if it > 0:  # the first pass warms up
            pre.append(e[0].elapsed_time(e[1]))
            dec.append(e[1].elapsed_time(e[2]))
    return {"prefill_ms": pre_ms, "decode_ms": dec_ms,
            "serial_prefill_ms": sum(pre) / len(pre), "serial_decode_ms": sum(dec) / len(dec),
            "h2d_bytes": h2d, "d2h_bytes": d2h}


# ------------------------------------------------------------- oracle (CPU) arm
_ORACLE_INPUTS: dict = {}


def oracle_sample(seconds: float, keep: bool = False):
    """Time the fp64 oracle on a bounded sample of the same step: rows of the long
    prefill spread over heads and positions, and whole decode sequences. Returns the
    measured TFLOP/s (prefill convention 4*D per visible key per row) and GB/s; with
    keep=True also the sampled rows and the oracle's outputs for them and for the
    decode. The inputs are drawn once per process."""
    import oracle
    if PREFILL.name not in _ORACLE_INPUTS:
        _ORACLE_INPUTS[PREFILL.name] = (inputs.make(PREFILL), inputs.make(DECODE))
    xp, xd = _ORACLE_INPUTS[PREFILL.name]
    L, D = PREFILL.Lq, PREFILL.D
    threads = oracle.default_threads()

    def rows_for(n):
        g = torch.Generator().manual_seed(7)
        heads = torch.randint(0, PREFILL.Hq, (n,), generator=g)
        pos = torch.randint(0, L, (n,), generator=g)
        if PREFILL.causal:
            vis = torch.clamp(pos + 1 + (PREFILL.Lk - PREFILL.Lq), min=0, max=PREFILL.Lk)
        else:
            vis = torch.full_like(pos, PREFILL.Lk)
        return (heads * L + pos).tolist(), int(vis.sum())

    # calibrate on samples that double until one takes a tenth of the budget, then size
    # the sample to about `seconds` of prefill work
    n = 64
    while True:
        rows, keys = rows_for(n)
        t = time.perf_counter()
        oracle.attn_fwd_rows(xp["q"], xp["k"], xp["v"], rows, PREFILL.scale, PREFILL.causal,
                             threads)
        dt = time.perf_counter() - t
        if dt >= 0.1 * seconds or n >= 100000:
            break
        n *= 2
    n = int(max(64, min(400000, n * (0.9 * seconds) / max(dt, 1e-4))))
    rows, keys = rows_for(n)
    t = time.perf_counter()
    ro, rl = oracle.attn_fwd_rows(xp["q"], xp["k"], xp["v"], rows, PREFILL.scale,
                                  PREFILL.causal, threads)
    t_pre = time.perf_counter() - t
    flops = 4.0 * D * keys
    t = time.perf_counter()
    do, dl = oracle.attn_paged(xd["q"], xd["k_cache"], xd["v_cache"], xd["block_table"],
                               xd["seq_lens"], DECODE.scale, threads)
    t_dec = time.perf_counter() - t
    nbytes = inputs.paged_bytes(DECODE, xd["seq_lens"])
    r = {"tflops": flops / t_pre / 1e12, "gbs": nbytes / t_dec / 1e9, "rows": n,
         "prefill_s": t_pre, "decode_s": t_dec, "threads": threads}
    if keep:
        r["prefill_ref"] = (rows, ro, rl)
        r["decode_ref"] = (do, dl)
    return r


O_TOL = {torch.float16: 2e-3, torch.bfloat16: 1.6e-2}
LSE_REL = 1e-4


def compare(out, lse, ro, rl, dtype, rows_note):
    """max |O err| and max lse error (|d| / max(1, |lse|)) of a GPU result against the
    oracle's, with the tolerances the parity tests use."""
    o = out.detach().to("cpu", torch.float64).reshape(ro.shape)
    err = float((o - ro).abs().max()) if ro.numel() else 0.0
    lg = lse.detach().to("cpu", torch.float64).reshape(rl.shape)
    fin = torch.isfinite(rl)
    same_inf = bool(torch.equal(torch.isfinite(lg), fin))
    lerr = float(((lg[fin] - rl[fin]).abs() / rl[fin].abs().clamp_min(1.0)).max()) if fin.any() else 0.0
    tol = O_TOL[dtype]
    return {"rows": rows_note, "max_abs_err": err, "tol": tol, "max_lse_rel_err": lerr,
            "lse_tol": LSE_REL, "ok": bool(err <= tol and lerr <= LSE_REL and same_inf)}


def cpu_baseline(seconds: float, gpu=None):
    """The oracle timed on the host cores on a bounded sample of the step (the CPU
    baseline). With the GPU results of the same inputs (`gpu`), the oracle's outputs for
    that sample are also compared with them: the long prefill on the sampled rows, the
    decode on every output, and the small dense workloads (timed in `configs`) on every
    output."""
    import oracle
    r = oracle_sample(seconds, keep=gpu is not None)
    line = {"value": r["tflops"], "unit": "TFLOP/s", "cores": r["threads"], "kind": "oracle",
            "sample": f"{r['rows']} random query rows of {PREFILL.name} (all their visible keys, "
                      f"{r['prefill_s']:.1f} s) + the whole {DECODE.name} decode "
                      f"({r['decode_s']:.2f} s, {r['gbs']:.3f} GB/s)",
            "paged_decode_gbs": r["gbs"]}
    if gpu is None:
        return line, None
    par = {}
    if gpu.get("prefill") is not None:
        rows, ro, rl = r["prefill_ref"]
        out, lse = gpu["prefill"]
        idx = torch.tensor(rows)
        par[PREFILL.name] = compare(out.reshape(-1, PREFILL.D)[idx.to(out.device)],
                                    lse.reshape(-1)[idx.to(lse.device)], ro, rl, PREFILL.dtype,
                                    f"{len(rows)} sampled rows (the CPU-baseline sample)")
    if gpu.get("decode") is not None:
        do, dl = r["decode_ref"]
        out, lse = gpu["decode"]
        par[DECODE.name] = compare(out, lse, do, dl, DECODE.dtype, "every output")
    for name, (x, out, lse) in gpu.get("configs", {}).items():
        spec = inputs.WORKLOADS[name]
        ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], spec.scale, spec.causal)
        par[name] = compare(out, lse, ro, rl, spec.dtype, "every output")
    return line, par


def run_reference(args, ws, rank):
    if rank != 0:
        return None
    # the whole run stays within a few minutes: cpu_seconds over all steps, with a small
    # floor per step (each step still runs the whole decode and some prefill rows)
    per_step = max(0.1, args.cpu_seconds / max(1, args.steps))
    for _ in range(min(args.warmup, 1)):
        oracle_sample(0.5)
    res = []
    t = time.perf_counter()
    for _ in range(args.steps):
        res.append(oracle_sample(per_step))
    total = time.perf_counter() - t
    tf = statistics.mean(r["tflops"] for r in res)
    gb = statistics.mean(r["gbs"] for r in res)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": tf,
        "unit": "TFLOP/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0,1) inputs shaped like the pages' workloads)",
        "config": {"workload": f"{PREFILL.name} + {DECODE.name}",
                   "note": "the fp64 CPU oracle on a bounded sample of each step"},
        "cpu_baseline": {"value": tf, "unit": "TFLOP/s", "cores": res[0]["threads"],
                         "kind": "oracle",
                         "sample": f"per step {res[0]['rows']} random prefill rows + the whole "
                                   f"decode workload"},
        "paged_decode": {"value": gb, "unit": "GB/s"},
        "e2e": {"value": tf, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU seconds for the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false",
                    help="skip the host-buffer end-to-end measurement (profiling runs)")
    ap.add_argument("--no-graphs", dest="graphs", action="store_false",
                    help="skip the CUDA-graph replay timing of the step's two calls")
    ap.add_argument("--no-fp8", dest="fp8", action="store_false",
                    help="skip the separately timed e4m3 forward of the prefill workload")
    ap.add_argument("--no-paged-prefill", dest="paged_prefill", action="store_false",
                    help="skip the separately timed paged-cache prefill of the prefill workload")
    ap.add_argument("--no-configs", dest="configs", action="store_false",
                    help="skip the separately timed small dense workloads (C1-C3 shapes)")
    ap.add_argument("--no-backward", dest="backward", action="store_false",
                    help="skip the separately timed backward pass of the prefill workload")
    ap.add_argument("--only", choices=["both", "prefill", "decode"], default="both",
                    help="run one kernel of the step only (profiling runs)")
    ap.add_argument("--copies", type=int, default=4,
                    help="device copies of the inputs the steps rotate over (4 > L2)")
    ap.add_argument("--window", type=int, nargs=2, metavar=("LEFT", "RIGHT"), default=None,
                    help="sliding window of the prefill call (-1 = unbounded side)")
    ap.add_argument("--prefill-workload", default=PREFILL_DEFAULT,
                    choices=[n for n, w in inputs.WORKLOADS.items() if w.kind == "dense"],
                    help="dense workload of the prefill call (default: the long causal prefill)")
    ap.add_argument("--decode-seqs", type=int, default=None,
                    help="the decode workload with this many sequences instead of 16 (same "
                         "length distribution, heads and seed): how its GB/s grows with the batch")
    args = ap.parse_args(argv)
    global PREFILL, DECODE
    PREFILL = inputs.WORKLOADS[args.prefill_workload]
    if args.decode_seqs is not None:
        if args.decode_seqs < 1:
            ap.error("--decode-seqs must be >= 1")
        DECODE = dataclasses.replace(DECODE, num_seqs=args.decode_seqs,
                                     name=DECODE.name.replace(f"_s{DECODE.num_seqs}_",
                                                              f"_s{args.decode_seqs}_"))
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    ws, rank, local = dist_env()
    if args.impl == "reference":
        line = run_reference(args, ws, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        line = run_ours(args, ws, rank, local)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

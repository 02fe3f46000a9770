"""Throughput of the quantized attention path on B200, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole path over one batch of synthetic input:
the quantize/smooth pass plus the fused INT8-QK / FP8-PV attention kernel
(``sage_attn``).  The default workload is the video-DiT long-sequence shape
B=1, H=24, N=32768, d=128, bf16, NHD, non-causal, K with a per-channel offset,
fp16+fp32 P.V accumulation (the largest of the five workloads, N >= 8K and
d = 128).  The image-DiT (B=2, H=24, N=4096, d=64) and causal GQA prefill
(B=4, Hq=32, Hkv=8, N=8192, d=128) workloads are measured in the same run and
reported under ``also``, each with its own roofline.

* ``value``: whole-job attention TOPS, 4*B*Hq*N^2*d (halved under the causal
  mask) per step, inputs resident in HBM, per-step CUDA events with an L2
  flush between steps (outside the events), max over ranks.
* ``roofline``: the fused attention kernel alone (sage_attn_quantized on the
  same buffers, per-launch CUDA events, L2 flushed) against the dense INT8/FP8
  tensor peak (2x the measured bf16 cuBLAS peak, the B200 nominal ratio); the
  tcgen05.mma rate this GPU measures for kind::i8 and kind::f8f6f4
  (sage_mma_probe) is reported beside it with the fraction against it.
* ``e2e``: the same metric through the public API (``sage_attn``) with pinned
  HOST buffers: every step uploads q, k, v and downloads its output inside the
  timed region.  ``value`` streams the steps (three CUDA streams, two device
  buffer sets: step i+1's upload and step i-1's download overlap step i);
  ``serial`` runs them one at a time with per-step events.
* ``cpu_baseline``: the CPU oracle on this host's cores, on a bounded sample of
  the same workload: exact fp64 attention of 512-row query chunks of successive
  heads (TOPS), and the quantization emulation of one head (GB/s).
* ``--impl reference``: there is no reference implementation to run; the
  reference arm times the CPU oracle (exact fp64 attention, bounded row
  samples) on the same workload instead.

Multi-GPU (torchrun): replicas only, one independent copy of the workload per
rank, no collective on the data path (weak scaling).
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "attention TOPS on 1 B200 (N=1K-32K, d=64/128) and % of dense INT8/FP8 tensor peak"
DEFAULT_WORKLOAD = W.VIDEO_DIT.name
ALSO = [W.IMAGE_DIT.name, W.LLM_GQA.name]
L2_FLUSH_BYTES = 256 << 20


def _traffic(workload: str):
    """DRAM bytes per launch of the fused kernel from the committed ncu capture, or None if the
    kernel source changed since the capture (or the workload was not captured)."""
    import hashlib
    try:
        kv = {}
        for line in open(os.path.join(ROOT, "profiles", "sage_fwd_traffic.txt")):
            line = line.strip()
            if line and not line.startswith("#") and "=" in line:
                k, v = line.split("=", 1)
                kv[k.strip()] = v.strip()
        src = open(os.path.join(ROOT, "quantized_attention_int8_b200", "csrc", "attn.cu"), "rb").read()
        if hashlib.sha256(src).hexdigest() != kv.get("attn_cu_sha256"):
            return None
        return int(kv[workload]) if workload in kv else None
    except (OSError, ValueError):
        return None


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return dict(bf16=float(m["bf16_tflops"]), bf16_sustained=float(m["bf16_tflops_sustained"]),
                    hbm=float(m["hbm_gbs"]), source="measured")
    except Exception:
        return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


# ------------------------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.dev = device_index
        self.out_path = os.path.join("/tmp", f"sage_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.out_path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.dev)], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return None
        rows = []
        for line in open(self.out_path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                rows.append(dict(sm=float(p[1]), smax=float(p[2]), power=float(p[3]), hw=p[5], hwt=p[6],
                                 swt=p[7], pcap=p[8]))
            except ValueError:
                continue
        if not rows:
            return None
        load = [r for r in rows if r["power"] > 200] or rows
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load)}


# ------------------------------------------------------------------------------------ timing
def _flush(buf):
    buf.add_(1)


HOST_AHEAD_CYCLES = 400_000  # ~0.2 ms of device-side sleep before each step's start event


def time_steps(fn, steps, warmup, flush_buf):
    """Per-step CUDA events on the current stream, L2 flushed before every step.

    A short device-side sleep sits between the flush and the start event, so the device is still
    busy while the host enqueues the step: the events then measure device time only, not the
    host's launch latency (as when a program enqueues its steps ahead of the device)."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        _flush(flush_buf)
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        _flush(flush_buf)
        torch.cuda._sleep(HOST_AHEAD_CYCLES)
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def time_e2e_streamed(qh, kh, vh, attn, steps, warmup, flush_buf):
    """Device time of `steps` end-to-end steps fed from pinned host memory: each step uploads
    q, k, v, runs `attn(q, k, v, out)` and downloads out, on three streams with two device
    buffer sets, so that uploads, compute and downloads of neighbouring steps overlap.  Events
    bracket the whole stream (first upload to last download); returns its milliseconds."""
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    nb = 2
    dev = [[torch.empty(t.shape, dtype=t.dtype, device="cuda") for t in (qh, kh, vh)] for _ in range(nb)]
    douts = [torch.empty(qh.shape, dtype=qh.dtype, device="cuda") for _ in range(nb)]
    houts = [torch.empty(qh.shape, dtype=qh.dtype).pin_memory() for _ in range(nb)]

    def run(n, start=None, end=None):
        up = [torch.cuda.Event() for _ in range(n)]
        done = [torch.cuda.Event() for _ in range(n)]
        down = [torch.cuda.Event() for _ in range(n)]
        if start is not None:
            start.record(s_in)
        for i in range(n):
            j = i % nb
            with torch.cuda.stream(s_in):
                if i >= nb:
                    s_in.wait_event(done[i - nb])  # buffer set j's inputs consumed
                for d, h in zip(dev[j], (qh, kh, vh)):
                    d.copy_(h, non_blocking=True)
                up[i].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(up[i])
                if i >= nb:
                    s_cmp.wait_event(down[i - nb])  # buffer set j's output read back
                _flush(flush_buf)
                attn(*dev[j], douts[j])
                done[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[i])
                houts[j].copy_(douts[j], non_blocking=True)
                down[i].record(s_out)
        if end is not None:
            end.record(s_out)  # after the last download, which follows every other step's work

    torch.cuda.synchronize()
    run(warmup)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(steps, a, b)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def _threads():
    try:
        import threadpoolctl
        return max([i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()] or [1])
    except Exception:
        return os.cpu_count()


def _head(t, layout, b, h):
    t = t[b:b + 1]
    return (t[:, h:h + 1] if layout == "HND" else t[:, :, h:h + 1]).contiguous()


def cpu_oracle_sample(w: W.Workload, q, k, v, budget_s: float, start: int = 0):
    """Exact fp64 attention (the oracle) of 512-row query chunks of successive (b=0, hq) heads, from
    chunk `start` on, until the time budget is used (at least one chunk).  Returns (TOPS, threads,
    rows, seconds, next start)."""
    from oracle import attention
    G = w.Hq // w.Hkv
    nchunk = (w.N + 511) // 512
    done, pairs, t0, i = 0, 0, time.perf_counter(), start
    while done == 0 or time.perf_counter() - t0 < budget_s:
        h, c = (i // nchunk) % w.Hq, i % nchunk
        rows = np.arange(c * 512, min(w.N, c * 512 + 512))
        qh, kh, vh = _head(q, w.layout, 0, h), _head(k, w.layout, 0, h // G), _head(v, w.layout, 0, h // G)
        attention.attention_f64(qh, kh, vh, w.layout, w.causal, W.sm_scale_of(w), heads=[(0, 0)], rows=rows)
        done += len(rows)
        pairs += int((rows + 1).sum()) if w.causal else len(rows) * w.N
        i += 1
    dt = time.perf_counter() - t0
    # the metric counts 4*d operations per visible (query, key) pair (causal: half of N^2 per head)
    ops = 4.0 * w.d * pairs
    return ops / dt / 1e12, _threads(), done, dt, i


def cpu_quantize_sample(w: W.Workload, q, k, v):
    """The quantization emulation (oracle) of one (b=0) kv head with its first query head: GB/s of
    the algorithmic bytes (2 B read + 1 B written per Q, K element; V 1 or 2 B written)."""
    from oracle import quant
    qh, kh, vh = _head(q, w.layout, 0, 0), _head(k, w.layout, 0, 0), _head(v, w.layout, 0, 0)
    t0 = time.perf_counter()
    quant.quantize(qh, kh, vh, w.layout, w.pv_mode, w.q_gran, w.smooth_v)
    dt = time.perf_counter() - t0
    n = qh.numel()
    nbytes = 3 * 2 * n + (4 if w.pv_mode & 2 else 3) * n
    return nbytes / dt / 1e9, dt


def job_throughput(local_ms: float, ops_per_step: float, steps: int, dist=None, device=None):
    """Whole-job TOPS for replicas: every rank ran `steps` steps of `ops_per_step` each in
    `local_ms`; the job's time is the slowest rank's (one MAX all-reduce of a scalar, outside
    the data path).  Returns (TOPS, max_ms)."""
    world = 1
    if dist is not None and dist.is_initialized():
        world = dist.get_world_size()
        t = torch.tensor([local_ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        local_ms = float(t.item())
    return world * ops_per_step * steps / (local_ms * 1e-3) / 1e12, local_ms


# ------------------------------------------------------------------------------------ arms
def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    q, k, v = W.make_inputs(w.with_(B=1))
    budget = args.ref_seconds / max(1, args.warmup + args.steps)  # split the run's CPU budget over its steps
    vals, start = [], 0
    for i in range(args.warmup + args.steps):
        tops, threads, rows, dt, start = cpu_oracle_sample(w, q, k, v, budget, start)
        if i >= args.warmup:
            vals.append((tops, rows, dt))
    val = statistics.median(t for t, _, _ in vals)
    ms = statistics.mean(dt for _, _, dt in vals) * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(w),
        "cpu_baseline": {"value": val, "unit": "TOPS", "cores": threads, "kind": "oracle",
                         "sample": f"exact fp64 attention of {vals[-1][1]} query rows (512-row chunks of successive "
                                   f"(b=0, hq) heads) of the workload per step, {budget:.1f} s budget"},
        "e2e": {"value": val, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "note": "no reference implementation exists for this path; the reference arm is the CPU oracle",
    }
    print(json.dumps(line), flush=True)


def _config(w):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "io_dtype": w.dtype,
            "layout": w.layout, "causal": w.causal, "pv_dtype": "fp16" if w.pv_mode & 2 else "fp8",
            "pv_accum": "fp16+fp32" if w.pv_mode & 1 else "fp32",
            "qk_quant_gran": {128: "per_block", 32: "per_warp", 1: "per_thread"}[w.q_gran], "smooth_v": w.smooth_v,
            "values": w.dist, "l2": "flushed between steps (256 MiB write outside the events)",
            "host": "each step enqueued while the device is busy (device sleep before the start event)"}


def _modes(w):
    pv = "fp16+fp32" if w.pv_mode & 1 else "fp32"
    pvd = "fp16" if w.pv_mode & 2 else "fp8"
    okw = dict(qk_quant_gran={128: "per_block", 32: "per_warp", 1: "per_thread"}[w.q_gran], smooth_v=w.smooth_v)
    return pv, pvd, okw


def _peak(w, peaks):
    if w.pv_mode & 2:
        # half the operations (Q.K^T) at the INT8 rate 2P, half (P.V, fp16) at the fp16 rate P:
        # the blended peak for all of them is 4P/3
        return 4.0 / 3.0 * peaks["bf16"], (f"4/3 x {peaks['source']} bf16 cuBLAS burst {peaks['bf16']} TF/s (half "
                                           "the operations at the INT8 rate 2x bf16, half at the fp16 rate 1x bf16)")
    return 2.0 * peaks["bf16"], (f"2 x {peaks['source']} bf16 cuBLAS burst {peaks['bf16']} TF/s "
                                 "(dense INT8/FP8 = 2x bf16 on B200)")


def mma_rates(qa, reps=5, iters=10000):
    """tcgen05.mma rate of this GPU per kind (sage_mma_probe: one CTA per SM issuing MMAs back to
    back), best of `reps` launches timed with CUDA events: TOPS for kind::i8 and kind::f8f6f4,
    TFLOP/s for kind::f16."""
    st = torch.cuda.current_stream()
    out = {}
    for kind, name in ((0, "i8"), (1, "f8f6f4"), (2, "f16")):
        ops = ctypes.c_double(0.0)
        best = 0.0
        for r in range(reps + 2):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            s = qa.capi.sage_mma_probe(kind, iters, ctypes.byref(ops), st.cuda_stream)
            b.record(st)
            if s != qa.SAGE_OK:
                raise RuntimeError(f"sage_mma_probe: {qa.sage_status_string(s)}")
            torch.cuda.synchronize()
            if r >= 2:
                best = max(best, ops.value / (a.elapsed_time(b) * 1e-3) / 1e12)
        out[name] = best
    qa.sage_check_status()
    return out


def measure(qa, w, args, flush, dist, rates, clk_sampler=None):
    """One workload: the whole path per step, the fused kernel alone, the quantize pass alone.
    Returns (result dict, device inputs, CPU inputs)."""
    pv, pvd, okw = _modes(w)
    scale = W.sm_scale_of(w)
    q, k, v = W.make_inputs(w)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out = torch.empty_like(qd)
    ops = w.ops()

    # ---- whole path (quantize + attention), device-resident inputs
    step = lambda: qa.sage_attn(qd, kd, vd, w.layout, w.causal, scale, pv, out=out, pv_dtype=pvd, **okw)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    if clk_sampler is not None:
        with clk_sampler:
            times = time_steps(step, args.steps, args.warmup, flush)
    else:
        times = time_steps(step, args.steps, args.warmup, flush)
    qa.sage_check_status()
    value, total_ms = job_throughput(sum(times), ops, args.steps, dist, "cuda")

    # ---- the fused attention kernel alone (roofline)
    z = qa.sage_quantize(qd, kd, vd, w.layout, pv, pvd, **okw)
    kern = lambda: qa.sage_attn_quantized(z, qd.dtype, w.layout, w.causal, scale, pv, out=out)
    ktimes = time_steps(kern, args.steps, args.warmup, flush)
    qa.sage_check_status()
    k_ms = statistics.mean(ktimes)
    peaks = _peaks()
    peak_tops, peak_src = _peak(w, peaks)
    achieved = ops / (k_ms * 1e-3) / 1e12
    # the same against the tcgen05.mma rate measured on this GPU: Q.K^T at the kind::i8 rate, P.V at
    # the kind::f8f6f4 (FP8 P.V) or kind::f16 (FP16 P.V) rate, half of the operations each
    pv_rate = rates["f16"] if w.pv_mode & 2 else rates["f8f6f4"]
    mma_peak = 1.0 / (0.5 / rates["i8"] + 0.5 / pv_rate)

    # ---- quantize pass alone (HBM-bound): algorithmic bytes = 2 B read + 1 B written per Q/K/V element
    # (V: 2 B written in the FP16 P.V modes); the C entry point on preallocated outputs, so the Python
    # allocations are not timed
    qopts = qa.opts(**okw)  # kept alive while qargs points at it
    qargs = [qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), w.B, w.Hq, w.Hkv, w.N, w.d,
             qa.SAGE_BF16 if qd.dtype == torch.bfloat16 else qa.SAGE_FP16,
             qa.SAGE_HND if w.layout == "HND" else qa.SAGE_NHD, w.pv_mode, ctypes.byref(qopts),
             *(z[n].data_ptr() for n in ("q8", "qs", "k8", "ks", "km", "v8t", "vs", "vm")),
             torch.cuda.current_stream().cuda_stream]
    qtimes = time_steps(lambda: qa.capi.sage_quantize(*qargs), max(3, args.steps // 2), 3, flush)
    qa.sage_check_status()
    q_ms = statistics.mean(qtimes)
    q_bytes = 3 * (q.numel() + k.numel()) + (4 if w.pv_mode & 2 else 3) * v.numel()
    del z
    res = {
        "value": value, "ms_per_step": total_ms / args.steps,
        "step_ms": {"min_ms": min(times), "median_ms": statistics.median(times), "max_ms": max(times)},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_tops, "unit": "TFLOP/s",
                     "frac": achieved / peak_tops, "traffic": _traffic(w.name),
                     "kernel": "sage_fwd_kernel", "kernel_ms": k_ms, "peak_source": peak_src,
                     "tcgen05_measured": {"peak": mma_peak, "frac": achieved / mma_peak,
                                          "rates": rates,
                                          "how": "sage_mma_probe (back-to-back tcgen05.mma, every SM) on this GPU; "
                                                 "half the operations at the kind::i8 rate, half at the P.V kind's "
                                                 "rate; frac above uses the bf16-derived peak"}},
        "quantize": {"ms": q_ms, "algorithmic_bytes": q_bytes, "GB_per_s": q_bytes / (q_ms * 1e-3) / 1e9,
                     "hbm_peak_GB_per_s": peaks["hbm"], "frac": q_bytes / (q_ms * 1e-3) / 1e9 / peaks["hbm"]},
        # d not in {64, 128, 256}: the kernels run on the zero-padded head dim
        "padded_work_value": value * qa.padded_dim(w.d) / w.d if qa.padded_dim(w.d) != w.d else None,
    }
    return res, (qd, kd, vd, out), (q, k, v)


def run_ours(args, w):
    import quantized_attention_int8_b200 as qa
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if not qa.sage_device_supported():
        raise SystemExit("this device is not a B200 (compute capability 10.0)")
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    rates = mma_rates(qa)
    clk = ClockSampler(torch.cuda.current_device())
    main_res, (qd, kd, vd, out), (q, k, v) = measure(qa, w, args, flush, dist, rates, clk)

    # ---- end to end through the public API with pinned host buffers
    pv, pvd, okw = _modes(w)
    scale = W.sm_scale_of(w)
    ops = w.ops()
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
    del qd, kd, vd
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    outh = torch.empty(q.shape, dtype=q.dtype).pin_memory()

    def e2e_step():
        a = qh.to("cuda", non_blocking=True)
        b = kh.to("cuda", non_blocking=True)
        c = vh.to("cuda", non_blocking=True)
        o = qa.sage_attn(a, b, c, w.layout, w.causal, scale, pv, pv_dtype=pvd, **okw)
        outh.copy_(o, non_blocking=True)

    # one step at a time (copy in, compute, copy out), per-step events: the latency of a call
    etimes = time_steps(e2e_step, args.steps, args.warmup, flush)
    serial_value, serial_ms = job_throughput(sum(etimes), ops, args.steps, dist, "cuda")
    # a stream of steps (the throughput of a job that feeds batches from host memory)
    e_ms = time_e2e_streamed(qh, kh, vh, lambda a, b, c, o: qa.sage_attn(a, b, c, w.layout, w.causal, scale, pv, out=o,
                                                                          pv_dtype=pvd, **okw),
                             args.steps, args.warmup, flush)
    e2e_value, e_ms = job_throughput(e_ms, ops, args.steps, dist, "cuda")
    qa.sage_check_status()
    del qh, kh, vh, outh
    torch.cuda.empty_cache()

    # ---- the other workloads, same measurements (no e2e)
    also = {}
    for name in ALSO:
        if name == w.name or args.no_also:
            continue
        res, dev, _ = measure(qa, W.BY_NAME[name], args, flush, dist, rates)
        res["config"] = _config(W.BY_NAME[name])
        also[name] = res
        del dev
        torch.cuda.empty_cache()

    if rank == 0:
        cpu = None
        if world == 1:
            tops, threads, rows, dt, _ = cpu_oracle_sample(w, q, k, v, 12.0)
            qgbs, qdt = cpu_quantize_sample(w, q, k, v)
            cpu = {"value": tops, "unit": "TOPS", "cores": threads, "kind": "oracle",
                   "sample": f"exact fp64 attention of {rows} query rows (512-row chunks of successive (b=0, hq) "
                             f"heads), {dt:.1f} s",
                   "quantize": {"value": qgbs, "unit": "GB/s", "kind": "oracle",
                                "sample": f"quantization emulation of one (b=0) head of Q, K and V, {qdt:.2f} s; "
                                          "bytes counted as for the GPU quantize pass"}}
        line = {
            "metric": METRIC, "value": main_res["value"], "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": main_res["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "i8+f16" if w.pv_mode & 2 else "i8+f8e4m3",
            "data": "synthetic",
            "config": _config(w),
            "roofline": main_res["roofline"],
            "quantize": main_res["quantize"],
            "cpu_baseline": cpu,
            "padded_work_value": main_res["padded_work_value"],
            "e2e": {"value": e2e_value, "unit": "TOPS", "h2d_bytes_per_step": in_bytes,
                    "d2h_bytes_per_step": out.numel() * out.element_size(), "ms_per_step": e_ms / args.steps,
                    "mode": "streamed: every step copies its q, k, v from pinned host memory and its output back "
                            "inside the timed region; step i+1's upload and step i-1's download overlap step i "
                            "(three streams, two device buffer sets, L2 flushed before each step's compute)",
                    "serial": {"value": serial_value, "ms_per_step": serial_ms / args.steps,
                               "mode": "one step at a time: upload, compute, download, per-step events"}},
            "step_ms": main_res["step_ms"],
            "gpu_launches": 4 * args.steps,
            "clocks": clk.summary(),
            "also": also,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.BY_NAME))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-also", action="store_true", help="measure only --workload")
    ap.add_argument("--ref-seconds", type=float, default=90.0,
                    help="reference arm: CPU seconds for the whole run (warm-up and timed steps)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    w = W.BY_NAME[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the Lightning Attention hot path on B200; prints ONE JSON line.

Headline workload (the configuration the metric is quoted on): bf16 prefill,
B=4, H=16, N=8192, d=128, blk=128, q,k ~ N(0,1/d), v ~ N(0,1), seed 0 (seed +
rank under torchrun).  A step is one la_prefill call over that batch, in the
schedule the library picks for it.  Inputs (384 MiB) and outputs exceed the
126 MB L2, so no flush is needed between steps.

  value     tokens/s of the whole job with inputs resident in HBM (max over ranks)
  e2e       the same metric through the public API with the inputs copied from
            pinned host memory and o/state copied back inside the timed region
  roofline  the dominant kernel (the prefill output pass; the variant the
            library dispatched is named) against measured HBM
            bandwidth: algorithmic bytes per launch / CUDA-event launch time
  secondary the backward of the headline prefill (dq, dk, dv), decode GB/s
            (128 seq x 64 heads, 256 steps) with the fp32 and the
            8-bit state (and a batch padded from 96 live rows to 128),
            long-context prefill (B=1, H=64, N=262144), the bf16 blk=64
            prefill and the packed varlen prefill where supported (single-GPU
            runs only)

``--impl reference`` times the fp64 CPU oracle (the reference arm of this
build) on a bounded sample of the same workload.

``--profile-case NAME`` runs one workload for --warmup + --steps calls with no
timing and prints a one-line summary: the command the ncu summaries under
profiles/ were captured with (prefill, prefill_blk64, decode, decode_q8,
long_prefill_32k, varlen_32k).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "lightning-attn prefill tokens/s & % bf16 tensor peak; decode HBM GB/s"
UNIT = "tokens/s"
B, H, N, D, BLK = 4, 16, 8192, 128, 128
BYTES_PER_TOKEN_HEAD = 8 * D                       # q,k,v read + o write, bf16
FLOPS_PER_TOKEN_HEAD = 4 * BLK * D + 4 * D * D     # dense-tile count (blk 128)
USEFUL_FLOPS_PER_TOKEN_HEAD = 2 * (BLK + 1) * D + 4 * D * D   # the causal half of the tile
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


# ----------------------------------------------------------------------------- env
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "prefill_seq_kernel_b4h16n8192.md")


def kernel_source_sha256(files=None) -> str:
    """Hash of the kernel sources (csrc/*.cuh, which hold every __global__ and
    __device__ function; or only the headers named in ``files``) without their
    comments and blank space: identifies the kernel version an ncu capture was
    taken of, so that an edit of a comment, or of another kernel's header,
    does not invalidate a capture.  lightning.cu (host-side validation,
    dispatch and launches) is not part of it."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "linear_attention_13_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(os.listdir(csrc)):
        if name.endswith(".cuh") and (files is None or name in files):
            with open(os.path.join(csrc, name), encoding="utf-8") as f:
                text = f.read()
            text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
            text = re.sub(r"//[^\n]*", " ", text)
            text = " ".join(text.split())
            h.update(name.encode() + b"\0" + text.encode())
    return h.hexdigest()


def captured_traffic(kernel: str, path: str = PROFILE_SUMMARY):
    """DRAM bytes (read + write) per launch of the headline kernel from the
    committed ncu summary, or None when the kernel sources changed since or
    the summary is of another kernel."""
    try:
        with open(path) as f:
            text = f.read()
    except OSError:
        return None
    fields = {}
    for line in text.splitlines():
        if ":" in line and line.startswith("- "):
            k, v = line[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    files = fields.get("source_files")
    files = set(files.split()) if files else None
    if fields.get("source_sha256") != kernel_source_sha256(files) or fields.get("kernel") != kernel:
        return None
    try:
        traffic = float(fields["traffic_bytes_per_launch"])
        traffic *= float(fields.get("traffic_scale_to_full", "1"))
        return int(traffic)
    except (KeyError, ValueError):
        return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS)


def line_roofline(kernel: str, alg_bytes: float, launch_ms: float, peaks, summary=None):
    """Roofline object of one kernel: algorithmic bytes of a launch over its
    average CUDA-event duration, against measured HBM bandwidth; ``traffic``
    from the committed ncu summary ``summary`` when it is of this kernel and
    of the current kernel sources (scaled to a full launch when the summary
    gives ``traffic_scale_to_full``), else null."""
    achieved = alg_bytes / (launch_ms / 1e3) / 1e9
    traffic = None
    if summary is not None:
        traffic = captured_traffic(kernel, os.path.join(ROOT, "profiles", summary))
    return {"bound": "hbm", "kernel": kernel, "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
            "peak_source": peaks["source"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": traffic, "algorithmic_bytes_per_launch": int(alg_bytes),
            "launch_ms": round(launch_ms, 5)}


class Dist:
    """One process per GPU (torchrun env); a no-op when WORLD_SIZE is 1.

    The backend is NCCL on GPUs; LA_DIST_BACKEND=gloo runs the same host
    logic (barrier, max over ranks) on CPU processes."""

    def __init__(self, backend=None):
        backend = backend or os.environ.get("LA_DIST_BACKEND", "nccl")
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.pg = None

    def init(self, device=None):
        if self.world > 1:
            import torch.distributed as dist
            kw = {}
            if self.backend == "nccl" and device is not None:
                kw["device_id"] = device
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, x: float, device=None) -> float:
        if self.pg is None:
            return float(x)
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()
            self.pg = None


class ClockSampler:
    """Samples SM clock, power and throttle reasons via NVML in a thread."""

    REASONS = {  # NVML clocks-event reason bits
        0x8: "hw_slowdown",
        0x40: "hw_thermal_slowdown",
        0x20: "sw_thermal_slowdown",
        0x4: "sw_power_cap",
    }

    def __init__(self, device_index: int, period_s: float = 0.05):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 - report instead of failing the bench
            self.error = repr(e)

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((sm, pw, rs))
            except Exception:  # noqa: BLE001
                pass
            self._stop.wait(self.period)

    def start(self):
        if self.handle is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
        return self.summary()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": getattr(self, "error", "no samples in the timed region")}
        reasons = set()
        for _, _, rs in self.samples:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons),
                "power_w_max": max(s[1] for s in self.samples),
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------- ours
def timed(stream, fn, steps, warmup, dist, device):
    """W untimed steps, then exactly `steps` timed between CUDA events on
    `stream`, bracketed by barrier + synchronize; returns max-over-ranks ms.
    (On a CPU device -- the multi-rank host tests -- a host clock stands in
    for the events.)"""
    import torch
    on_gpu = getattr(device, "type", str(device)) == "cuda"
    sync = torch.cuda.synchronize if on_gpu else (lambda: None)
    for _ in range(warmup):
        fn()
    sync()
    dist.barrier()
    sync()
    if on_gpu:
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
    else:
        t0 = time.perf_counter()
    for _ in range(steps):
        fn()
    if on_gpu:
        end.record(stream)
    sync()
    ms = start.elapsed_time(end) if on_gpu else (time.perf_counter() - t0) * 1e3
    dist.barrier()
    return dist.max(ms, device)


def job_throughput(units_per_rank_step: float, steps: int, max_ms: float, world: int) -> float:
    """Whole-job throughput under weak scaling: every rank processes the same
    number of units per step; the job takes the slowest rank's time."""
    return world * units_per_rank_step * steps / (max_ms / 1e3)


def kernel_times(la):
    out = {}
    for kid in range(la.LA_NUM_KERNEL_IDS):
        st, ms, n = la.la_timing_read(kid)
        if st == la.LA_OK and n > 0:
            out[la.la_kernel_name(kid)] = {"total_ms": ms, "launches": n}
    return out


def bench_ours(args, dist):
    import torch
    import linear_attention_13_b200 as la
    from linear_attention_13_b200 import build as labuild
    from linear_attention_13_b200 import inputs

    labuild.build()
    device = torch.device("cuda", dist.local_rank)
    torch.cuda.set_device(device)
    dist.init(device)
    peaks = load_peaks()
    stream = torch.cuda.current_stream()

    q, k, v = inputs.qkv((B, H, N, D), dtype=torch.bfloat16, device=device, seed=dist.rank)
    o = torch.empty_like(q)
    st = torch.empty((B, H, D, D), dtype=torch.float32, device=device)

    def step():
        la.prefill(q, k, v, blk=BLK, out=o, state_out=st)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    if la.la_get_last_error() != la.LA_OK:
        raise RuntimeError("prefill reported a device error")

    sampler = ClockSampler(dist.local_rank).start()
    la.la_timing_enable(args.steps * 4 + 64)
    ms = timed(stream, step, args.steps, args.warmup, dist, device)
    clocks = sampler.stop()
    ktimes = kernel_times(la)
    la.la_timing_enable(0)
    if la.la_get_last_error() != la.LA_OK:
        raise RuntimeError("prefill reported a device error in the timed region")

    ms_step = ms / args.steps
    tokens_step = B * N
    value = job_throughput(tokens_step, args.steps, ms, dist.world)
    flops_step = B * H * N * FLOPS_PER_TOKEN_HEAD
    bytes_step = B * H * N * BYTES_PER_TOKEN_HEAD
    # launches during the timed region = totals minus warm-up launches (the
    # timing pool was enabled for warm-up + timed steps)
    launches_total = sum(v["launches"] for v in ktimes.values())
    launches_timed = launches_total * args.steps // (args.steps + args.warmup)

    main = ktimes.get("prefill_main", {"total_ms": float("nan"), "launches": 1})
    main_kernel = la.la_prefill_main_kernel()
    main_ms = main["total_ms"] / max(main["launches"], 1)
    achieved = bytes_step / (main_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": main_kernel, "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "peak_source": peaks["source"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": captured_traffic(main_kernel),
                "algorithmic_bytes_per_launch": bytes_step,
                "launch_ms": round(main_ms, 5)}
    step_tflops = flops_step / (ms_step / 1e3) / 1e12
    tensor = {"tflops": round(step_tflops, 2), "peak_tflops": peaks["bf16_tflops"],
              "frac_of_peak": round(step_tflops / peaks["bf16_tflops"], 4),
              "flops_per_token_head": FLOPS_PER_TOKEN_HEAD,
              "useful_tflops": round(step_tflops * USEFUL_FLOPS_PER_TOKEN_HEAD / FLOPS_PER_TOKEN_HEAD, 2),
              "useful_frac_of_peak": round(step_tflops * USEFUL_FLOPS_PER_TOKEN_HEAD / FLOPS_PER_TOKEN_HEAD /
                                           peaks["bf16_tflops"], 4),
              "useful_flops_per_token_head": USEFUL_FLOPS_PER_TOKEN_HEAD,
              "step_hbm_frac": round(bytes_step / (ms_step / 1e3) / 1e9 / peaks["hbm_gbs"], 4)}

    e2e = bench_e2e(args, dist, device, stream, q, k, v)

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "prefill bf16 B=4 H=16 N=8192 d=128 blk=128",
                   "global_batch": B * dist.world, "seq_len": N, "heads": H, "head_dim": D,
                   "blk": BLK, "parallelism": f"dp{dist.world}" if dist.world > 1 else "single",
                   "l2": "inputs (384 MiB) larger than L2; no flush"},
        "roofline": roofline,
        "tensor": tensor,
        "kernels": {k_: {"avg_ms": round(v_["total_ms"] / max(v_["launches"], 1), 5),
                         "launches": v_["launches"]} for k_, v_ in ktimes.items()},
        "gpu_launches": launches_timed,
        "clocks": clocks,
        "e2e": e2e,
    }
    del q, k, v, o, st
    torch.cuda.empty_cache()
    if dist.world == 1 and not args.no_secondary:
        result["secondary"] = bench_secondary(args, device, stream, peaks)
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_budget)
        if "secondary" in result:
            sec = result["secondary"]
            budget = max(1.0, args.cpu_budget / 3)
            sec["long_prefill"]["cpu_baseline"] = cpu_baseline_long(budget)
            sec["decode"]["cpu_baseline"] = cpu_baseline_decode(budget)
            sec["varlen_prefill"]["cpu_baseline"] = cpu_baseline_varlen(budget)
    return result


def bench_e2e(args, dist, device, stream, qd, kd, vd):
    """Same metric through the public API with host buffers: every step copies
    q, k, v from pinned host memory, runs la_prefill and copies o and the state
    back.  The copies run on their own streams, so step i+1's upload and step
    i-1's download overlap step i's kernel (two device buffer sets); the timed
    region holds every step's copies and ends when the last download has
    landed."""
    import torch
    import linear_attention_13_b200 as la
    hq, hk, hv = (t.to("cpu").pin_memory() for t in (qd, kd, vd))
    ho = torch.empty(qd.shape, dtype=qd.dtype).pin_memory()
    hs = torch.empty((B, H, D, D), dtype=torch.float32).pin_memory()
    sets = [{"q": torch.empty_like(qd), "k": torch.empty_like(qd), "v": torch.empty_like(qd),
             "o": torch.empty_like(qd),
             "s": torch.empty((B, H, D, D), dtype=torch.float32, device=device)} for _ in range(2)]
    s_h2d = torch.cuda.Stream(device)
    s_d2h = torch.cuda.Stream(device)
    s_cmp = stream
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(nsteps):
        for i in range(nsteps):
            b = i & 1
            st = sets[b]
            if i >= 2:
                s_h2d.wait_event(ev_done[b])      # step i-2 no longer reads these inputs
            with torch.cuda.stream(s_h2d):
                st["q"].copy_(hq, non_blocking=True)
                st["k"].copy_(hk, non_blocking=True)
                st["v"].copy_(hv, non_blocking=True)
                ev_in[b].record(s_h2d)
            s_cmp.wait_event(ev_in[b])
            if i >= 2:
                s_cmp.wait_event(ev_out[b])       # step i-2's outputs have been copied out
            la.prefill(st["q"], st["k"], st["v"], blk=BLK, out=st["o"], state_out=st["s"], stream=s_cmp)
            ev_done[b].record(s_cmp)
            s_d2h.wait_event(ev_done[b])
            with torch.cuda.stream(s_d2h):
                ho.copy_(st["o"], non_blocking=True)
                hs.copy_(st["s"], non_blocking=True)
                ev_out[b].record(s_d2h)

    steps = max(3, min(args.steps, args.e2e_steps))
    run(3)
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(s_h2d)
    run(steps)
    end.record(s_d2h)
    torch.cuda.synchronize()
    dist.barrier()
    ms = dist.max(start.elapsed_time(end), device)
    if la.la_get_last_error() != la.LA_OK:
        raise RuntimeError("prefill reported a device error in the end-to-end run")
    h2d = 3 * qd.numel() * qd.element_size()
    d2h = ho.numel() * ho.element_size() + hs.numel() * 4
    return {"value": round(job_throughput(B * N, steps, ms, dist.world), 1), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 4),
            "pipelining": "uploads, kernel and downloads on separate streams, two buffer sets"}


def bench_secondary(args, device, stream, peaks):
    import torch
    import linear_attention_13_b200 as la
    from linear_attention_13_b200 import inputs

    class _Solo:
        world = 1

        def barrier(self):
            pass

        def max(self, x, device=None):
            return x

    solo = _Solo()
    out = {}

    # -- the headline prefill with 64-token blocks (B=4 H=16 N=8192 d=128 blk=64)
    q, k, v = inputs.qkv((B, H, N, D), dtype=torch.bfloat16, device=device, seed=0)
    o = torch.empty_like(q)
    st = torch.empty((B, H, D, D), dtype=torch.float32, device=device)
    n64 = 200
    la.la_timing_enable(n64 * 4 + 64)
    ms = timed(stream, lambda: la.prefill(q, k, v, blk=64, out=o, state_out=st), n64, 5, solo, device)
    kt = kernel_times(la)
    la.la_timing_enable(0)
    main64 = kt.get("prefill_main", {"total_ms": float("nan"), "launches": 1})
    k_ms = main64["total_ms"] / max(main64["launches"], 1)
    kern64 = la.la_prefill_main_kernel()
    out["prefill_blk64"] = {
        "roofline": line_roofline(kern64, B * H * N * BYTES_PER_TOKEN_HEAD, k_ms, peaks,
                                  "prefill_seq64_kernel_b4h16n8192.md" if kern64 == "prefill_seq64_kernel" else None),
        "workload": f"prefill bf16 B={B} H={H} N={N} d={D} blk=64",
        "tokens_per_s": round(B * N / (ms / n64 / 1e3), 1), "ms_per_step": round(ms / n64, 5),
        "hbm_frac": round(B * H * N * BYTES_PER_TOKEN_HEAD / (k_ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
        "tensor_frac": round(B * H * N * (4 * 64 * D + 4 * D * D) / (ms / n64 / 1e3) / 1e12 /
                             peaks["bf16_tflops"], 4),
        "kernels": {k_: round(v_["total_ms"] / max(v_["launches"], 1), 5) for k_, v_ in kt.items()}}
    del q, k, v, o, st
    torch.cuda.empty_cache()

    # -- backward of the same prefill (dq, dk, dv of sum(dO * o)), blk=128
    q, k, v = inputs.qkv((B, H, N, D), dtype=torch.bfloat16, device=device, seed=0)
    do = inputs.qkv((B, H, N, D), dtype=torch.bfloat16, device=device, seed=1)[2]
    grads = tuple(torch.empty_like(q) for _ in range(3))
    la.la_timing_enable(64 * 8)
    nb = 20
    ms = timed(stream, lambda: la.prefill_backward(q, k, v, do, blk=BLK, out=grads), nb, 3, solo, device)
    kt = kernel_times(la)
    la.la_timing_enable(0)
    bytes_bwd = B * H * N * 7 * D * 2      # q, k, v, dO read; dq, dk, dv written (bf16)
    out["backward"] = {
        "roofline": dict(line_roofline("prefill_seq_kernel (three launches: dq causal, dk and dv "
                                       "anti-causal)", bytes_bwd, ms / nb, peaks),
                         note="whole backward step (its three launches) against 1792 B per token-head"),
        "workload": f"prefill backward bf16 B={B} H={H} N={N} d={D} blk=128 (dq, dk, dv)",
        "ms_per_step": round(ms / nb, 5),
        "tokens_per_s": round(B * N / (ms / nb / 1e3), 1),
        "hbm_frac": round(bytes_bwd / (ms / nb / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
        "algorithmic_bytes": bytes_bwd,
        "kernels": {k_: [v_["launches"] // nb, round(v_["total_ms"] / max(v_["launches"], 1), 5)]
                    for k_, v_ in kt.items()}}
    del q, k, v, do, grads
    torch.cuda.empty_cache()

    # -- decode: 128 sequences x 64 heads, d=128; state from a 4096-token prefill
    n_seq, Hd, N0, steps = 128, 64, 4096, 256
    q0, k0, v0 = inputs.qkv((n_seq, Hd, N0, D), dtype=torch.bfloat16, device=device, seed=0)
    S = torch.empty((n_seq, Hd, D, D), dtype=torch.float32, device=device)
    o0 = torch.empty_like(q0)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    la.prefill(q0, k0, v0, blk=BLK, out=o0, state_out=S)
    t1.record(stream)
    torch.cuda.synchronize()
    pre_ms = t0.elapsed_time(t1)
    out["decode_init_prefill"] = {
        "workload": "prefill bf16 B=128 H=64 N=4096 d=128 (decode initial state, one call)",
        "tokens_per_s": round(n_seq * N0 / (pre_ms / 1e3), 1), "ms": round(pre_ms, 3),
        "hbm_frac": round(n_seq * Hd * N0 * BYTES_PER_TOKEN_HEAD / (pre_ms / 1e3) / 1e9 /
                          peaks["hbm_gbs"], 4)}
    del q0, k0, v0, o0
    torch.cuda.empty_cache()
    step_inputs = [inputs.decode_step_inputs(n_seq, Hd, D, s, device=device)
                   for s in range(1, steps + 1)]
    od = torch.empty((n_seq, Hd, D), dtype=torch.bfloat16, device=device)
    it = iter(range(10 ** 9))

    def dstep():
        i = next(it) % steps
        qq, kk, vv = step_inputs[i]
        la.decode_step(qq, kk, vv, S, out=od)

    la.la_timing_enable(steps + 64)
    ms = timed(stream, dstep, steps, 5, solo, device)
    kt = kernel_times(la)
    la.la_timing_enable(0)
    dec = kt.get("decode_step_kernel", {"total_ms": float("nan"), "launches": 1})
    k_ms = dec["total_ms"] / max(dec["launches"], 1)
    bytes_step = n_seq * Hd * (8 * D * D + 8 * D)
    out["decode"] = {
        "roofline": line_roofline("decode_step_kernel", bytes_step, k_ms, peaks,
                                  "decode_step_kernel_128x64.md"),
        "workload": "decode step, 128 seq x 64 heads, d=128, fp32 state, 256 steps",
        "ms_per_step": round(ms / steps, 5), "GB/s": round(bytes_step / (ms / steps / 1e3) / 1e9, 1),
        "kernel_GB/s": round(bytes_step / (k_ms / 1e3) / 1e9, 1),
        "hbm_frac": round(bytes_step / (k_ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
        "bytes_per_step": bytes_step}

    # -- the same decode on the 8-bit state (int8 codes + one fp32 scale per
    #    key row), all 128 rows live, then a batch padded from 96 live rows to
    #    a 128-row level through the slot pool
    codes, scales = la.state_quantize_q8(S)
    del S
    torch.cuda.empty_cache()

    def qstep(slots=None):
        i = next(it) % steps
        qq, kk, vv = step_inputs[i]
        la.decode_step_q8(qq, kk, vv, codes, scales, slots, out=od)

    la.la_timing_enable(steps + 64)
    ms = timed(stream, qstep, steps, 5, solo, device)
    kt = kernel_times(la)
    la.la_timing_enable(0)
    dec = kt.get("decode_step_kernel", {"total_ms": float("nan"), "launches": 1})
    k_ms = dec["total_ms"] / max(dec["launches"], 1)
    bytes_q8 = n_seq * Hd * (2 * (D * D + 4 * D) + 8 * D)
    padded = torch.tensor(list(range(96)) + [-1] * 32, dtype=torch.int32, device=device)
    la.la_timing_enable(steps + 64)
    ms_pad = timed(stream, lambda: qstep(padded), steps, 5, solo, device)
    kt_pad = kernel_times(la)
    la.la_timing_enable(0)
    dec_pad = kt_pad.get("decode_step_kernel", {"total_ms": float("nan"), "launches": 1})
    out["decode_q8"] = {
        "roofline": line_roofline("decode_step_q8_kernel", bytes_q8, k_ms, peaks,
                                  "decode_step_q8_kernel_128x64.md"),
        "workload": "decode step, 128 seq x 64 heads, d=128, 8-bit state (int8 + fp32 row scales), "
                    "256 steps",
        "ms_per_step": round(ms / steps, 5), "kernel_ms": round(k_ms, 5),
        "kernel_GB/s": round(bytes_q8 / (k_ms / 1e3) / 1e9, 1),
        "hbm_frac": round(bytes_q8 / (k_ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
        "bytes_per_step": bytes_q8,
        "speedup_vs_fp32_state_kernel": round(out["decode"]["bytes_per_step"] /
                                              out["decode"]["kernel_GB/s"] / 1e9 / (k_ms / 1e3), 3),
        "padded_96_of_128_kernel_ms": round(dec_pad["total_ms"] / max(dec_pad["launches"], 1), 5)}
    del step_inputs, codes, scales, od
    torch.cuda.empty_cache()

    # -- long-context prefill B=1 H=64 N=262144
    Hl, Nl = 64, 262144
    q, k, v = inputs.qkv((1, Hl, Nl, D), dtype=torch.bfloat16, device=device, seed=0)
    o = torch.empty_like(q)
    st = torch.empty((1, Hl, D, D), dtype=torch.float32, device=device)
    la.la_timing_enable(64)
    ms = timed(stream, lambda: la.prefill(q, k, v, blk=BLK, out=o, state_out=st), 5, 2, solo, device)
    kt = kernel_times(la)
    la.la_timing_enable(0)
    bytes_step = Hl * Nl * BYTES_PER_TOKEN_HEAD
    main_l = kt.get("prefill_main", {"total_ms": float("nan"), "launches": 1})
    out["long_prefill"] = {
        "roofline": line_roofline(la.la_prefill_main_kernel(), bytes_step,
                                  main_l["total_ms"] / max(main_l["launches"], 1), peaks,
                                  "prefill_seq_kernel_long_b1h64n262144.md"),
        "workload": "prefill bf16 B=1 H=64 N=262144 d=128 blk=128",
        "tokens_per_s": round(Nl / (ms / 5 / 1e3), 1), "ms_per_step": round(ms / 5, 4),
        "hbm_frac": round(bytes_step / (ms / 5 / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
        "tensor_frac": round(Hl * Nl * FLOPS_PER_TOKEN_HEAD / (ms / 5 / 1e3) / 1e12 /
                             peaks["bf16_tflops"], 4),
        "kernels": {k_: round(v_["total_ms"] / max(v_["launches"], 1), 4) for k_, v_ in kt.items()}}
    del q, k, v, o, st
    torch.cuda.empty_cache()

    # -- packed variable-length prefill: 2^20 tokens, lengths U[1024, 65536], H=64
    Tv, Hv = 1 << 20, 64
    lens = inputs.varlen_lengths(Tv, 1024, 65536, seed=0)
    cu = torch.from_numpy(inputs.cu_seqlens_from_lengths(lens)).to(device)
    q, k, v = inputs.qkv((Hv, Tv, D), dtype=torch.bfloat16, device=device, seed=0)
    o = torch.empty_like(q)
    st = torch.empty((len(lens), Hv, D, D), dtype=torch.float32, device=device)
    la.la_timing_enable(64)
    ms = timed(stream, lambda: la.prefill_varlen(q, k, v, cu, blk=BLK, out=o, state_out=st), 3, 2,
               solo, device)
    kt = kernel_times(la)
    la.la_timing_enable(0)
    bytes_step = Hv * Tv * BYTES_PER_TOKEN_HEAD
    main_v = kt.get("prefill_main", {"total_ms": float("nan"), "launches": 1})
    out["varlen_prefill"] = {
        "roofline": line_roofline(la.la_prefill_main_kernel(), bytes_step,
                                  main_v["total_ms"] / max(main_v["launches"], 1), peaks,
                                  "prefill_tc_kernel_varlen_t2p20.md"),
        "workload": f"packed prefill bf16 T=2^20 ({len(lens)} sequences, lengths U[1024,65536] "
                    "seed 0), H=64, d=128, blk=128",
        "tokens_per_s": round(Tv / (ms / 3 / 1e3), 1), "ms_per_step": round(ms / 3, 4),
        "hbm_frac": round(bytes_step / (ms / 3 / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
        "kernels": {k_: round(v_["total_ms"] / max(v_["launches"], 1), 4) for k_, v_ in kt.items()}}
    del q, k, v, o, st
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- profiling
PROFILE_CASES = {
    "prefill": "prefill bf16 B=4 H=16 N=8192 d=128 blk=128 (the headline launch)",
    "prefill_blk64": "prefill bf16 B=4 H=16 N=8192 d=128 blk=64",
    "decode": "decode step, 128 seq x 64 heads, d=128, fp32 state (random state)",
    "decode_q8": "decode step, 128 seq x 64 heads, d=128, 8-bit state (random state, quantised)",
    "long_prefill_32k": "prefill bf16 B=1 H=64 N=32768 d=128 blk=128 (long-context shape, "
                        "1/8 of the length)",
    "varlen_32k": "packed prefill bf16 T=2^15, lengths U[1024,8192] seed 0, H=64, d=128",
    "varlen_2heads": "packed prefill bf16 T=2^20, lengths U[1024,65536] seed 0 (the packed "
                     "configuration's sequences), H=2, d=128, one chunk per sequence (the schedule "
                     "the 64-head configuration runs)",
    "backward": "prefill backward bf16 B=4 H=16 N=8192 d=128 blk=128 (dq causal, dk and dv "
                "anti-causal launches)",
}


def profile_case(args):
    """Launch one workload --warmup + --steps times, untimed, for an ncu capture."""
    import torch
    import linear_attention_13_b200 as la
    from linear_attention_13_b200 import inputs

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    name = args.profile_case
    if name in ("prefill", "prefill_blk64", "long_prefill_32k"):
        shape = (B, H, N, D) if name != "long_prefill_32k" else (1, 64, 32768, D)
        blk = 64 if name == "prefill_blk64" else BLK
        q, k, v = inputs.qkv(shape, dtype=torch.bfloat16, device=device, seed=0)
        o = torch.empty_like(q)
        st = torch.empty(shape[:2] + (D, D), dtype=torch.float32, device=device)

        def call():
            la.prefill(q, k, v, blk=blk, out=o, state_out=st)
    elif name == "decode":
        n_seq, Hd = 128, 64
        S = torch.randn((n_seq, Hd, D, D), dtype=torch.float32, device=device)
        qq, kk, vv = inputs.decode_step_inputs(n_seq, Hd, D, 1, device=device)
        od = torch.empty((n_seq, Hd, D), dtype=torch.bfloat16, device=device)

        def call():
            la.decode_step(qq, kk, vv, S, out=od)
    elif name == "decode_q8":
        n_seq, Hd = 128, 64
        codes, scales = la.state_quantize_q8(
            torch.randn((n_seq, Hd, D, D), dtype=torch.float32, device=device))
        qq, kk, vv = inputs.decode_step_inputs(n_seq, Hd, D, 1, device=device)
        od = torch.empty((n_seq, Hd, D), dtype=torch.bfloat16, device=device)

        def call():
            la.decode_step_q8(qq, kk, vv, codes, scales, out=od)
    elif name == "varlen_2heads":
        Tv, Hv = 1 << 20, 2
        lens = inputs.varlen_lengths(Tv, 1024, 65536, seed=0)
        cu = torch.from_numpy(inputs.cu_seqlens_from_lengths(lens)).to(device)
        q, k, v = inputs.qkv((Hv, Tv, D), dtype=torch.bfloat16, device=device, seed=0)
        o = torch.empty_like(q)
        st = torch.empty((len(lens), Hv, D, D), dtype=torch.float32, device=device)

        def call():
            la.prefill_varlen(q, k, v, cu, blk=BLK, out=o, state_out=st, chunk_tokens=Tv,
                              flags=la.LA_FLAG_FUSED)
    elif name == "backward":
        q, k, v = inputs.qkv((B, H, N, D), dtype=torch.bfloat16, device=device, seed=0)
        do = inputs.qkv((B, H, N, D), dtype=torch.bfloat16, device=device, seed=1)[2]
        grads = tuple(torch.empty_like(q) for _ in range(3))

        def call():
            la.prefill_backward(q, k, v, do, blk=BLK, out=grads)
    elif name == "varlen_32k":
        Tv, Hv = 1 << 15, 64
        lens = inputs.varlen_lengths(Tv, 1024, 8192, seed=0)
        cu = torch.from_numpy(inputs.cu_seqlens_from_lengths(lens)).to(device)
        q, k, v = inputs.qkv((Hv, Tv, D), dtype=torch.bfloat16, device=device, seed=0)
        o = torch.empty_like(q)
        st = torch.empty((len(lens), Hv, D, D), dtype=torch.float32, device=device)

        def call():
            la.prefill_varlen(q, k, v, cu, blk=BLK, out=o, state_out=st)
    else:
        raise SystemExit(f"unknown profile case {name}")
    for _ in range(args.warmup + args.steps):
        call()
    torch.cuda.synchronize()
    status = la.la_get_last_error()
    print(json.dumps({"profile_case": name, "workload": PROFILE_CASES[name],
                      "calls": args.warmup + args.steps, "status": status}), flush=True)
    return 0 if status == la.LA_OK else 1


# ----------------------------------------------------------------------------- oracle
def cpu_baseline(budget_s: float = 15.0):
    """The fp64 oracle (recurrent form, OpenMP over heads) on a bounded sample
    of the headline workload: whole 8192-token heads, as many as fit the time
    budget; tokens/s = token-heads/s / H."""
    import torch
    import oracle
    from linear_attention_13_b200 import inputs
    cores = oracle.num_threads()
    q, k, v = inputs.qkv((1, cores, N, D), dtype=torch.bfloat16, device="cpu", seed=0)
    q, k, v = (t.to(torch.float64).numpy() for t in (q, k, v))
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.prefill_recurrent(q, k, v)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    token_heads = reps * cores * N
    return {"value": round(token_heads / dt / H, 1), "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": f"{reps} x {cores} heads of N={N}, d={D} (fp64 recurrent form), "
                      f"{dt:.1f} s; tokens/s = token-heads/s / H ({H})"}


def _oracle_rate(run, budget_s):
    """Repeat ``run`` (returns the token-heads it processed) for about
    ``budget_s`` seconds; returns (token-heads per second, reps, seconds)."""
    t0 = time.perf_counter()
    done = reps = 0
    while True:
        done += run()
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return done / dt, reps, dt


def cpu_baseline_long(budget_s: float = 5.0):
    """The fp64 oracle on 4 sampled heads of the long-context prefill (B=1,
    H=64, N=262144, d=128), on a token prefix sized to the time budget; the
    full-configuration time is extrapolated from the measured rate."""
    import torch
    import oracle
    from linear_attention_13_b200 import inputs
    Hl, Nl, heads = 64, 262144, 4
    q, k, v = inputs.qkv((1, heads, 2048, D), dtype=torch.bfloat16, device="cpu", seed=0)
    q, k, v = (t.to(torch.float64).numpy() for t in (q, k, v))
    t0 = time.perf_counter()
    oracle.prefill_recurrent(q, k, v)
    per_token = (time.perf_counter() - t0) / 2048
    n_tok = int(min(Nl, max(2048, budget_s / max(per_token, 1e-9) / 2)))
    q, k, v = inputs.qkv((1, heads, n_tok, D), dtype=torch.bfloat16, device="cpu", seed=0)
    q, k, v = (t.to(torch.float64).numpy() for t in (q, k, v))
    rate, reps, dt = _oracle_rate(lambda: (oracle.prefill_recurrent(q, k, v), heads * n_tok)[1], budget_s)
    return {"value": round(rate / Hl, 1), "unit": UNIT, "cores": min(heads, oracle.num_threads()),
            "kind": "oracle", "token_heads_per_s": round(rate, 1),
            "extrapolated_full_config_s": round(Hl * Nl / rate, 1),
            "sample": f"{reps} x {heads} sampled heads x {n_tok} tokens of B=1 H=64 N=262144 d=128 "
                      f"(fp64 recurrent form, one thread per head), {dt:.1f} s; tokens/s = "
                      f"token-heads/s / 64; full-configuration time extrapolated"}


def cpu_baseline_decode(budget_s: float = 5.0):
    """The fp64 oracle on the decode configuration (128 sequences x 64 heads,
    d=128): one all-head step, and 16 sampled (sequence, head) trajectories of a
    4096-token prefill plus 256 steps."""
    import numpy as np
    import torch
    import oracle
    from linear_attention_13_b200 import inputs
    n_seq, Hd, N0, steps = 128, 64, 4096, 256
    rng = np.random.default_rng(0)
    S = rng.standard_normal((n_seq, Hd, D, D))
    qq, kk, vv = (t.to(torch.float64).numpy() for t in inputs.decode_step_inputs(n_seq, Hd, D, 1))
    t0 = time.perf_counter()
    oracle.decode_step(qq, kk, vv, S)
    step_s = time.perf_counter() - t0
    del S
    # 16 trajectories: prefill of 4096 tokens, then 256 single-token steps
    q, k, v = inputs.qkv((1, 16, N0, D), dtype=torch.bfloat16, device="cpu", seed=0)
    q, k, v = (t.to(torch.float64).numpy() for t in (q, k, v))
    t0 = time.perf_counter()
    _, st = oracle.prefill_recurrent(q, k, v)
    for s_ in range(1, steps + 1):
        a, b_, c = (t.to(torch.float64).numpy() for t in inputs.qkv((1, 16, D), dtype=torch.bfloat16, seed=s_))
        _, st = oracle.decode_step(a, b_, c, st)
    traj_s = time.perf_counter() - t0
    head_steps = n_seq * Hd
    return {"value": round(head_steps / step_s, 1), "unit": "head-steps/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "state_GB_per_s_fp32_equivalent": round(head_steps * 8 * D * D / step_s / 1e9, 2),
            "all_head_step_s": round(step_s, 3),
            "trajectories_s": round(traj_s, 2),
            "extrapolated_256_steps_s": round(steps * step_s, 1),
            "sample": "one step of all 128 x 64 heads (fp64 states), plus 16 sampled (sequence, head) "
                      "trajectories of a 4096-token prefill and 256 steps; 256-step time extrapolated"}


def cpu_baseline_varlen(budget_s: float = 5.0):
    """The fp64 oracle on 8 sampled heads of the packed prefill (T=2^20,
    lengths U[1024, 65536] seed 0, H=64, d=128), over the first packed
    sequences that fit the time budget; the full time is extrapolated."""
    import numpy as np
    import torch
    import oracle
    from linear_attention_13_b200 import inputs
    Tv, Hv, heads = 1 << 20, 64, 8
    lens = inputs.varlen_lengths(Tv, 1024, 65536, seed=0)
    # token budget from a short probe, then whole leading sequences
    q, k, v = inputs.qkv((heads, 2048, D), dtype=torch.bfloat16, device="cpu", seed=0)
    q, k, v = (t.to(torch.float64).numpy() for t in (q, k, v))
    t0 = time.perf_counter()
    oracle.prefill_varlen(q, k, v, np.array([0, 2048], dtype=np.int32))
    per_token = (time.perf_counter() - t0) / 2048
    want = int(budget_s / max(per_token, 1e-9) / 2)
    take, acc = [], 0
    for n in lens:
        if acc and acc + n > want:
            break
        take.append(n)
        acc += n
    cu = inputs.cu_seqlens_from_lengths(take)
    q, k, v = inputs.qkv((heads, acc, D), dtype=torch.bfloat16, device="cpu", seed=0)
    q, k, v = (t.to(torch.float64).numpy() for t in (q, k, v))
    rate, reps, dt = _oracle_rate(lambda: (oracle.prefill_varlen(q, k, v, cu), heads * acc)[1], budget_s)
    return {"value": round(rate / Hv, 1), "unit": UNIT, "cores": min(heads, oracle.num_threads()),
            "kind": "oracle", "token_heads_per_s": round(rate, 1),
            "extrapolated_full_config_s": round(Hv * Tv / rate, 1),
            "sample": f"{reps} x {heads} sampled heads x the first {len(take)} packed sequences "
                      f"({acc} tokens) of T=2^20, H=64, d=128 (fp64 recurrent form per sequence), "
                      f"{dt:.1f} s; tokens/s = token-heads/s / 64; full time extrapolated"}


def bench_reference(args, dist):
    """Reference arm: the fp64 CPU oracle, as it stands, on host cores."""
    import torch
    import oracle
    from linear_attention_13_b200 import inputs
    cores = oracle.num_threads()
    # size one step so that warm-up + timed steps stay within ~2 minutes
    step_budget = max(0.05, args.ref_budget / max(args.steps + args.warmup, 1))
    q, k, v = inputs.qkv((1, cores, N, D), dtype=torch.bfloat16, device="cpu", seed=0)
    q, k, v = (t.to(torch.float64).numpy() for t in (q, k, v))
    t0 = time.perf_counter()
    oracle.prefill_recurrent(q[:, :, :512], k[:, :, :512], v[:, :, :512])
    per_token = (time.perf_counter() - t0) / 512
    n_tok = int(max(128, min(N, step_budget / max(per_token, 1e-9))))
    qs, ks, vs = q[:, :, :n_tok].copy(), k[:, :, :n_tok].copy(), v[:, :, :n_tok].copy()
    for _ in range(args.warmup):
        oracle.prefill_recurrent(qs, ks, vs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.prefill_recurrent(qs, ks, vs)
    dt = time.perf_counter() - t0
    value = args.steps * cores * n_tok / dt / H
    sample = (f"each step: {cores} heads x {n_tok} tokens of the N={N}, d={D} workload "
              f"(fp64 recurrent oracle); tokens/s = token-heads/s / H ({H})")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT,
            "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "prefill bf16 B=4 H=16 N=8192 d=128 blk=128 (sampled)",
                       "global_batch": B, "seq_len": N},
            "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=120.0,
                    help="seconds of oracle work for the whole --impl reference run")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES), default=None)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.profile_case is not None:
        return profile_case(args)
    dist = Dist()
    if args.impl == "reference":
        if dist.rank != 0:
            return 0
        print(json.dumps(bench_reference(args, dist)), flush=True)
        return 0
    res = bench_ours(args, dist)
    if dist.rank == 0:
        print(json.dumps(res), flush=True)
    dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())

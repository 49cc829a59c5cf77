#!/usr/bin/env python
"""Benchmark of the wave-round hot path on B200.

A step is one wave round of a streaming rollout at the Wan2.1-1.3B shape
(12 heads x 128, 30x52 tokens per frame, 3-frame chunks of 4680 tokens,
7 cache chunks, 4 in-round chunks at staggered noise levels): host plan,
RoPE/append of the round's new Q/K/V into the ring pool, and block-causal
attention.  The ring advances one chunk per step.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Multi-GPU runs are independent replicas (the path has no exchange step): each
rank runs its own rollout; the value is the work of all ranks divided by the
slowest rank's device time.  The reference arm (--impl reference) times the
CPU oracle on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time
from typing import Optional

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "chunk-causal attn TFLOP/s & wave rounds/s at Wan-1.3B shape; % BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("wf", "reference", "library"), default="wf",
                    help="library: context only -- library Blackwell attention kernels on the same work")
    ap.add_argument("--config", default="wan13b_round")
    ap.add_argument("--scores", choices=("bf16", "fp8"), default="bf16",
                    help="fp8: e4m3 Q/K codes with block scales (quantization timed with RoPE/append)")
    ap.add_argument("--fused-q-rope", action="store_true",
                    help="the attention rotates the raw Q itself; the append pass writes only K'/V")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--soak", type=float, default=0.0,
                    help="seconds of untimed steps right before the timed region, so that the board "
                         "reaches its power-capped steady clock (default 0: timed right after warm-up)")
    ap.add_argument("--no-fp8-side", action="store_true",
                    help="skip the side measurement of the 8-bit score variant on a 16-bit run")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha(read=None):
    """Hash of the attention kernel's code (line comments and blank lines
    dropped, so that editing a comment does not orphan a capture)."""
    h = hashlib.sha256()
    for name in ("attn_sm100.cu", "sm100_ptx.cuh", "rope_math.cuh", "wf_plan.h", "wf_plan.cpp"):
        if read is None:
            with open(os.path.join(ROOT, "chunk_causal_attention_block_b200", "csrc", name)) as f:
                text = f.read()
        else:
            text = read(name)
        for line in text.splitlines():
            code = line.split("//", 1)[0].rstrip()
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def dram_traffic(config):
    """Per-launch DRAM bytes of the attention kernel from the committed ncu summary,
    or None when the kernel source changed since that capture."""
    path = os.path.join(ROOT, "profiles", "attn_dram_traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("kernel_source_sha") != kernel_source_sha():
        return None
    return t.get("bytes_per_launch", {}).get(config)


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Largest value over all ranks (the device time of the slowest replica)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(rank: int) -> int:
    """Each replica draws its own inputs: seed 42 (the plugin's base_seed) + rank."""
    return 42 + rank


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock, power and clock-event reasons sampled DURING the timed region.

    NVML is polled in a thread every ~2 ms and each sample is timestamped, so
    that only the samples inside [t0, t1] (host times bracketing the timed
    region: the queue is empty at t0 and drained at t1) are summarised; a
    timed region of ~100 ms then still yields dozens of samples.  Without
    NVML it falls back to `nvidia-smi -lms 200` over the whole window."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (nvmlClocksEventReason*)
    REASON_BITS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
                   ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80))
    PERIOD_S = 0.002

    def __init__(self, gpu_index: int, uuid: Optional[str] = None):
        self.gpu = gpu_index
        self.uuid = uuid
        self.proc = None
        self.path = None
        self.nvml = None
        self.handle = None
        self.rows = []
        self.thread = None
        self.stop_flag = False

    def _open_nvml(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            handle = None
            if self.uuid:
                try:
                    handle = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + self.uuid)
                except Exception:  # noqa: BLE001 - fall back to the index
                    handle = None
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.nvml, self.handle = pynvml, handle
            return True
        except Exception:  # noqa: BLE001 - no NVML: use nvidia-smi
            return False

    def _poll(self):
        nv, h = self.nvml, self.handle
        smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop_flag:
            try:
                row = (time.perf_counter(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), smax,
                       nv.nvmlDeviceGetPowerUsage(h) / 1000.0, nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                self.rows.append(row)
            except Exception:  # noqa: BLE001 - a failed query skips one sample
                pass
            time.sleep(self.PERIOD_S)

    def start(self):
        self.rows = []
        if self._open_nvml():
            self.stop_flag = False
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        fd, self.path = tempfile.mkstemp(prefix="wf_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.gpu)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    @classmethod
    def summarise(cls, rows, t0=None, t1=None):
        """rows: (time, sm_mhz, sm_max_mhz, power_w, reason_bits).  Summary of
        the rows inside [t0, t1] (all rows if no window is given)."""
        inside = [r for r in rows if (t0 is None or r[0] >= t0) and (t1 is None or r[0] <= t1)]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [r[1] for r in inside]
        bits = 0
        for r in inside:
            bits |= int(r[4])
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": max(r[2] for r in inside),
                "power_w_median": round(statistics.median(r[3] for r in inside), 1),
                "reasons": sorted(n for n, bit in cls.REASON_BITS if bits & bit),
                "samples": len(inside), "source": f"NVML every {1e3 * cls.PERIOD_S:.0f} ms inside the timed region"}

    def stop(self, t0=None, t1=None):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=10)
            self.thread = None
            return self.summarise(self.rows, t0, t1)
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        smax = max(float(r[2]) for r in rows)
        loaded = [s for s, r in zip(sm, rows) if float(r[3]) > 200.0] or sm
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows), "source": "nvidia-smi every 200 ms over the whole window"}


# ------------------------------------------------------------------ oracle (CPU) sample

def oracle_sample(cfg, seconds: float, first_n0: int, n0: int, seed: int = 42):
    """Time the CPU oracle on a bounded sample of one round: whole heads, a
    fixed set of query rows per chunk, every visible key (with its RoPE).
    Returns (algorithmic flops done, seconds, description)."""
    import numpy as np
    from tests import gpu_common as gc

    rows_per_chunk = min(256, cfg.C)
    rows = np.concatenate([i * cfg.C + np.arange(rows_per_chunk) for i in range(cfg.R)])
    flops_per_head = sum(4.0 * cfg.D * rows_per_chunk * k for k in cfg.visible_keys())
    done, heads, t_total = 0.0, 0, 0.0
    while t_total < seconds and heads < cfg.H:
        arrays = gc.oracle_inputs(cfg, n0, first_n0, [heads], seed=seed)  # drawing is not timed
        t0 = time.perf_counter()
        gc.oracle_call(cfg, n0, arrays, rows=rows)
        t_total += time.perf_counter() - t0
        done += flops_per_head
        heads += 1
    desc = (f"oracle wave_round (fp64 NumPy) on {heads} head(s) x {rows_per_chunk} query rows per in-round "
            f"chunk of round n0={n0}, all visible keys incl. their RoPE; input drawing excluded")
    return done, t_total, desc


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ------------------------------------------------------------------ arms

def run_reference(args, rank, world):
    """CPU oracle arm: rank 0 only, K timed steps of a bounded oracle sample."""
    if rank != 0:
        return None
    import numpy as np  # noqa: F401
    from chunk_causal_attention_block_b200.rollout import CONFIGS

    cfg = CONFIGS[args.config]
    # each step is a bounded sample (at least one head) so that the run stays within a few minutes
    per_step = max(0.5, 120.0 / max(1, args.steps + args.warmup))
    for w in range(args.warmup):
        oracle_sample(cfg, 0.1, cfg.Wc, cfg.Wc + w)
    flops, secs = 0.0, 0.0
    desc = ""
    for s in range(args.steps):
        f, t, desc = oracle_sample(cfg, per_step, cfg.Wc, cfg.Wc + args.warmup + s)
        flops += f
        secs += t
    value = flops / secs / 1e12
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Irwin-Hall(12) N(0,1) draws, seed 42)",
        "config": {"workload": cfg.name + " (oracle sample per step)", "heads": cfg.H, "head_dim": cfg.D,
                   "chunk_tokens": cfg.C, "cache_chunks": cfg.Wc, "inround_chunks": cfg.R,
                   "parallelism": f"replicas x{args.gpus} (reference arm runs on rank 0 only)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def fp8_side(cfg, dev, stream, rank, world, W, K):
    """The same rounds with 8-bit (e4m3) scores, device-timed like the main
    run (plan, RoPE/append, both quantizations, attention per step; inputs
    drawn on the device before timing), so that one default run records both
    variants.  Returns the summary for the JSON line."""
    import torch
    from chunk_causal_attention_block_b200 import wf
    from chunk_causal_attention_block_b200.rollout import Rollout

    ro = Rollout(cfg, device=dev, want_lse=False, seed=replica_seed(rank), fp8=True)
    ro.prefill()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    # inputs are drawn per round on the device; only plan + kernels are timed
    for r in range(W):
        ro.fill_inputs(ro.n0_of(r), cfg.R, r)
        ro.plan_round(r)
        ro.append()
        ro.attend()
    torch.cuda.synchronize()
    step_ms = []
    for s in range(K):
        r = W + s
        ro.fill_inputs(ro.n0_of(r), cfg.R, r)
        ev[s][0].record(stream)
        ro.plan_round(r)
        ro.append()
        ev[s][1].record(stream)
        ro.attend()
        ev[s][2].record(stream)
    torch.cuda.synchronize()
    code, detail = ro.device_status()
    if code != wf.WF_OK:
        raise RuntimeError(f"device status (8-bit scores) {wf.status_string(code)} {detail}")
    attn = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    step = statistics.mean(e[0].elapsed_time(e[2]) for e in ev)
    attn = max_over_ranks(attn, world, dev)
    step = max_over_ranks(step, world, dev)
    flops = cfg.attn_flops()
    return {"attn_tflops_kernel": flops / (attn / 1e3) / 1e12, "step_tflops": flops * world / (step / 1e3) / 1e12,
            "attn_ms": attn, "ms_per_step": step, "steps": K, "warmup": W,
            "dtype": "e4m3 scores, bf16 P/V/O", "gpu_launches": 4 * K,
            "timing": "device events per step around plan+RoPE/append+quantize and attention; "
                      "input drawing between steps is outside them"}


def run_wf(args, rank, world, local_rank):
    import numpy as np  # noqa: F401
    import torch
    import torch.distributed as dist

    from chunk_causal_attention_block_b200 import wf
    from chunk_causal_attention_block_b200.rollout import CONFIGS, Rollout

    wf.lib()  # fails loudly if the CUDA library is missing
    cfg = CONFIGS[args.config]
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    W, K = args.warmup, args.steps
    ro = Rollout(cfg, device=dev, want_lse=False, seed=replica_seed(rank), fp8=args.scores == "fp8",
                 fused_q_rope=args.fused_q_rope)
    ro.prefill()
    first_n0, n0_first = ro.first_n0, ro.n0_of(0)  # the oracle sample's round

    # every step's inputs resident in HBM before timing (round r draws tag r)
    tdt = torch.bfloat16 if cfg.dtype == wf.WF_BF16 else torch.float32
    nq = cfg.R * cfg.C
    inputs = []
    for r in range(W + K):
        q, k, v = (torch.empty(nq, cfg.H, cfg.D, dtype=tdt, device=dev) for _ in range(3))
        for t, dst in ((wf.WF_SYNTH_Q, q), (wf.WF_SYNTH_K, k), (wf.WF_SYNTH_V, v)):
            wf.wf_synth_fill(dst, cfg.dtype, ro.seed, t, r, ro.n0_of(r), cfg.R, cfg.C, cfg.H, cfg.D,
                             kscale=(cfg.kscale and t == wf.WF_SYNTH_K), stream=stream)
        inputs.append((q, k, v))
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]

    def step(r, events=None):
        ro.q, ro.k, ro.v = inputs[r]
        ro.plan_round(r)
        if events:
            events[0].record(stream)
        ro.append()
        if events:
            events[1].record(stream)
        ro.attend()
        if events:
            events[2].record(stream)

    for r in range(W):
        step(r)
    soak_steps = 0
    if args.soak > 0:  # untimed steps over the warm-up rounds until the time is up
        t_soak = time.perf_counter() + args.soak
        while time.perf_counter() < t_soak:
            step(soak_steps % W)
            soak_steps += 1
            if soak_steps % 4 == 0:
                torch.cuda.synchronize()  # keep the host within a few steps of the device
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]),
                           uuid=str(getattr(props, "uuid", "") or "") or None)
    sampler.start()
    if sampler.thread is None:
        time.sleep(0.3)  # nvidia-smi's first sample
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    host_t0 = time.perf_counter()
    t_start.record(stream)
    for s in range(K):
        step(W + s, ev[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    host_t1 = time.perf_counter()
    clocks = sampler.stop(host_t0, host_t1)
    # host time of planning one round (wf_plan_round without the device copy),
    # reported beside the device-timed step
    plan_host = torch.empty(wf.wf_plan_bytes(ro.desc(ro.n0_of(W + K))), dtype=torch.uint8)
    plan_ts = []
    for r in range(10):
        t0 = time.perf_counter()
        wf.wf_plan_round(ro.desc(ro.n0_of(W + K + r)), plan_host)
        plan_ts.append(time.perf_counter() - t0)
    plan_ms = 1e3 * statistics.median(plan_ts)
    ms = t_start.elapsed_time(t_end)
    rope_ms = [e[0].elapsed_time(e[1]) for e in ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    code, detail = ro.device_status()
    if code != wf.WF_OK:
        raise RuntimeError(f"device status {wf.status_string(code)} {detail}")
    ms_max = max_over_ranks(ms, world, dev)

    # End-to-end through the public calls with host buffers: every step copies
    # its Q/K/V from pinned host memory to the device and reads O back, inside
    # the timed region.  Copies run on their own streams, double-buffered, so
    # the upload of step r+1 and the read-back of step r-1 overlap step r's
    # kernels; events order every buffer reuse.  Each round's plan is built
    # and copied on the upload stream with its inputs (two host and two
    # device plan buffers): a plan copy queued on the compute stream would
    # wait behind the 57 MB input uploads on the same copy engine.
    e2e = None
    if not args.no_e2e:
        nsets = min(4, W + K)
        host_in = [tuple(x.cpu().pin_memory() for x in inputs[i]) for i in range(nsets)]
        host_out = [torch.empty(nq, cfg.H, cfg.D, dtype=tdt).pin_memory() for _ in range(2)]
        dev_in = [tuple(torch.empty_like(inputs[0][0]) for _ in range(3)) for _ in range(2)]
        dev_out = [torch.empty(nq, cfg.H, cfg.D, dtype=tdt, device=dev) for _ in range(2)]
        plan_bytes = max(wf.wf_plan_bytes(ro.desc(ro.n0_of(r))) for r in range(2 * (W + K) + 1))
        host_plan = [torch.empty(plan_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]
        dev_plan = [torch.empty(plan_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
        del inputs
        torch.cuda.empty_cache()
        up = torch.cuda.Stream(dev)
        down = torch.cuda.Stream(dev)
        in_free = [torch.cuda.Event() for _ in range(2)]     # attention done with a set (inputs, plan)
        in_ready = [torch.cuda.Event() for _ in range(2)]    # upload of a set (plan + inputs) done
        out_ready = [torch.cuda.Event() for _ in range(2)]   # attention wrote an output buffer
        out_free = [torch.cuda.Event() for _ in range(2)]    # read-back of an output buffer done

        def upload(r):
            b = r % 2
            in_ready[b].synchronize()  # the host plan buffer's previous copy has left
            up.wait_event(in_free[b])
            wf.wf_plan_round(ro.desc(ro.n0_of(r)), host_plan[b], dev_plan[b], up)
            with torch.cuda.stream(up):
                for dst, src in zip(dev_in[b], host_in[r % nsets]):
                    dst.copy_(src, non_blocking=True)
            in_ready[b].record(up)

        def compute(r):
            b = r % 2
            stream.wait_event(in_ready[b])
            ro.q, ro.k, ro.v = dev_in[b]
            ro.host_plan, ro.dev_plan = host_plan[b], dev_plan[b]
            ro.append()
            stream.wait_event(out_free[b])
            ro.out = dev_out[b]
            ro.attend()
            in_free[b].record(stream)
            out_ready[b].record(stream)

        def download(r):
            b = r % 2
            down.wait_event(out_ready[b])
            with torch.cuda.stream(down):
                host_out[b].copy_(dev_out[b], non_blocking=True)
            out_free[b].record(down)

        def run(first, count):
            upload(first)
            for s in range(count):
                if s + 1 < count:
                    upload(first + s + 1)
                compute(first + s)
                download(first + s)

        base = W + K
        run(base, W)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(up)
        run(base + W, K)
        stream.wait_stream(down)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        elem = 2 if cfg.dtype == wf.WF_BF16 else 4
        e2e = {"value": cfg.attn_flops() * K * world / (e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": 3 * nq * cfg.H * cfg.D * elem + wf.wf_plan_bytes(ro.desc(ro.n0_of(base + W))),
               "d2h_bytes_per_step": nq * cfg.H * cfg.D * elem,
               "ms_per_step": e_ms / K,
               "overlap": "plan + uploads of step r+1 and read-back of step r-1 overlap step r on two copy streams"}
        code, detail = ro.device_status()
        if code != wf.WF_OK:
            raise RuntimeError(f"device status {wf.status_string(code)} {detail}")

    side = None
    if args.scores == "bf16" and cfg.dtype == wf.WF_BF16 and not args.fused_q_rope and not args.no_fp8_side:
        side = fp8_side(cfg, dev, stream, rank, world, W, K)

    if rank != 0:
        return None
    peaks, peak_kind = load_peaks()
    flops = cfg.attn_flops()
    attn_avg = statistics.mean(attn_ms)
    rope_avg = statistics.mean(rope_ms)
    # the append pass moves Q, K, V in and Q', K', V out; K and V only when Q's RoPE is fused
    rope_bytes = cfg.rope_bytes() * (4 if args.fused_q_rope else 6) // 6
    achieved = flops / (attn_avg / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])
    traffic = dram_traffic(args.config)
    value = flops * K * world / (ms_max / 1e3) / 1e12
    elem = 2 if cfg.dtype == wf.WF_BF16 else 4
    # RoPE/append + attention, the combine pass of split units, the two quantizations of the 8-bit path
    launches_per_step = 2 + (1 if wf.decode_plan(ro.host_plan)["key_parts"] > 1 else 0) + \
        (2 if args.scores == "fp8" else 0)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("e4m3 scores, bf16 P/V/O" if args.scores == "fp8" else "bf16") if cfg.dtype == wf.WF_BF16
        else "f32",
        "data": "synthetic (seeded Irwin-Hall(12) N(0,1) draws, seed 42 + rank, drawn on device before timing)",
        "config": {"workload": cfg.name, "heads": cfg.H, "head_dim": cfg.D,
                   "tokens_per_frame": cfg.fh * cfg.fw, "chunk_tokens": cfg.C, "cache_chunks": cfg.Wc,
                   "inround_chunks": cfg.R, "queries_per_round": nq,
                   "visible_keys_per_chunk": cfg.visible_keys(), "global_batch": world,
                   "parallelism": f"replicas x{world}",
                   "l2": (f"inputs larger than L2 (per-round Q/K/V {cfg.rope_bytes() / 2 / 1e6:.0f} MB, "
                          f"K/V pool {2 * cfg.slots * cfg.C * cfg.H * cfg.D * elem / 1e6:.0f} MB, "
                          "fresh inputs each step)")},
        "wave_rounds_per_s": K * world / (ms_max / 1e3),
        "plan_ms_host": plan_ms,
        "attn_tflops_kernel": achieved,
        "pct_bf16_peak": {"of_spec_2250": 100 * achieved / 2250.0,
                          f"of_{peak_kind}_burst": 100 * achieved / peak,
                          f"of_{peak_kind}_sustained": 100 * achieved / float(peaks["bf16_tflops_sustained"])},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "attn_fwd_sm100", "peak_kind": f"{peak_kind} bf16 burst"},
        "rope_append": {"ms": rope_avg, "gb_s": rope_bytes / (rope_avg / 1e3) / 1e9,
                        "frac_of_hbm": rope_bytes / (rope_avg / 1e3) / 1e9 / float(peaks["hbm_gbs"]),
                        "bytes": rope_bytes, "fused_q_rope": args.fused_q_rope},
        "attn_ms": attn_avg,
        "gpu_launches": launches_per_step * K,
        "clocks": clocks,
        "e2e": e2e,
        **({"soak": {"seconds": args.soak, "steps": soak_steps}} if args.soak > 0 else {}),
    }
    if side is not None:
        line["fp8_scores"] = side
    if world == 1 and not args.no_cpu_baseline:
        f, t, desc = oracle_sample(cfg, args.cpu_seconds, first_n0, n0_first)
        line["cpu_baseline"] = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
                                "kind": "oracle", "sample": desc, "seconds": t}
    return line


def run_library(args, rank):
    """Context arm, never the product path: the round's attention work (each
    in-round chunk's queries against its visible keys, no mask inside,
    bf16) run through two library Blackwell attention kernels from
    flashinfer -- the TRT-LLM-gen context kernel (paged K/V) and the CuTe-DSL
    prefill kernel -- device-timed like the main arm, on rank 0 only."""
    if rank != 0:
        return None
    import torch
    from chunk_causal_attention_block_b200.rollout import CONFIGS
    cfg = CONFIGS[args.config]
    line = {"impl": "library", "metric": METRIC, "unit": "TFLOP/s", "config": {"workload": cfg.name},
            "note": "context only: library kernels on the same work, not this library's path"}
    if not torch.cuda.is_available():
        line["unavailable"] = "no CUDA device"
        return line
    try:
        import flashinfer  # noqa: F401
    except Exception as e:  # noqa: BLE001 - report and stop
        line["unavailable"] = f"flashinfer not importable: {e!r}"[:200]
        return line
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    H, D, C = cfg.H, cfg.D, cfg.C
    kv = [int(x) for x in cfg.visible_keys()]
    nq, nk = cfg.R * C, sum(kv)
    flops = cfg.attn_flops()
    g = torch.Generator(device=dev)
    g.manual_seed(42)
    q = torch.randn(nq, H, D, device=dev, dtype=torch.bfloat16, generator=g)
    qo = torch.tensor([i * C for i in range(cfg.R + 1)], dtype=torch.int32, device=dev)
    kvp = torch.tensor([0] + [sum(kv[:i + 1]) for i in range(len(kv))], dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(D)
    W, K = args.warmup, args.steps
    stream = torch.cuda.current_stream(dev)
    uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", "") or "") or None

    def timed(fn):
        for _ in range(W):
            fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        sampler = ClockSampler(0, uuid=uuid)
        sampler.start()
        t0 = time.perf_counter()
        for a, b in ev:
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        clocks = sampler.stop(t0, time.perf_counter())
        ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
        return {"attn_tflops_kernel": flops / (ms / 1e3) / 1e12, "attn_ms": ms, "clocks": clocks}

    kernels = {}
    try:
        from flashinfer.prefill import trtllm_batch_context_with_kv_cache
        page = 64
        pages = [(x + page - 1) // page for x in kv]
        kc = torch.randn(sum(pages), H, page, D, device=dev, dtype=torch.bfloat16, generator=g)
        vc = torch.randn(sum(pages), H, page, D, device=dev, dtype=torch.bfloat16, generator=g)
        bt = torch.zeros(len(kv), max(pages), dtype=torch.int32, device=dev)
        off = 0
        for i, n in enumerate(pages):
            bt[i, :n] = torch.arange(off, off + n, dtype=torch.int32, device=dev)
            off += n
        lens = torch.tensor(kv, dtype=torch.int32, device=dev)
        ws = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)
        out = torch.empty(nq, H, D, device=dev, dtype=torch.bfloat16)
        kernels["trtllm_gen_context"] = timed(lambda: trtllm_batch_context_with_kv_cache(
            q, (kc, vc), ws, bt, lens, C, max(kv), scale, 1.0, len(kv), qo, kvp, out=out, kv_layout="HND",
            causal=False))
        kernels["trtllm_gen_context"]["layout"] = f"paged K/V, HND, page {page}"
        del kc, vc, ws
    except Exception as e:  # noqa: BLE001 - a kernel the installed library lacks is reported, not fatal
        kernels["trtllm_gen_context"] = {"unavailable": repr(e)[:200]}
    try:
        from flashinfer.cute_dsl.attention.wrappers.batch_prefill import BatchPrefillCuteDSLWrapper
        k = torch.randn(nk, H, D, device=dev, dtype=torch.bfloat16, generator=g)
        v = torch.randn(nk, H, D, device=dev, dtype=torch.bfloat16, generator=g)
        w = BatchPrefillCuteDSLWrapper(torch.empty(16 << 20, dtype=torch.uint8, device=dev))
        w.plan(qo, kvp, H, H, D, causal=False, sm_scale=scale, q_data_type=torch.bfloat16,
               kv_data_type=torch.bfloat16)
        o2 = torch.empty(nq, H, D, device=dev, dtype=torch.bfloat16)
        kernels["cute_dsl_prefill"] = timed(lambda: w.run(q, k, v, out=o2))
        kernels["cute_dsl_prefill"]["note"] = "run() includes its copy of O into the caller's tensor"
    except Exception as e:  # noqa: BLE001
        kernels["cute_dsl_prefill"] = {"unavailable": repr(e)[:200]}
    line.update({"steps": K, "warmup": W, "kernels": kernels})
    return line


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "library":
        line = run_library(args, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    if args.impl == "reference":
        # the oracle arm is CPU-only; under torchrun only rank 0 works
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_wf(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

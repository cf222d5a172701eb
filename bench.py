#!/usr/bin/env python3
"""Benchmark of the quantized attention forward on B200.

One step = one full forward (statistics + quantize + fused attention) of the
workload, through the C ABI (sage_attn_fwd).  Metric: TOPS = 4*B*H*N^2*d / t.

  python bench.py [--gpus N --steps K --warmup W] [--workload flux|video|...]
  python bench.py --shard ...            # one problem split by heads over the GPUs
  python bench.py --impl reference ...   # the CPU oracle, timed on the host

N > 1 GPUs (torchrun): every rank runs its own copy of the workload (the heads
of independent problems; no data-path collective), so the scaling is weak and
the value is the sum over ranks of the work divided by the slowest rank's time.

With --shard the ranks instead split ONE problem by heads (each rank computes
its heads on strided views of the shared input) and all-gather the bf16
outputs over NCCL, so the scaling is strong; the time of a step covers the
kernels and the gather.

Inputs are seeded synthetic tensors (quantized_attention_qk_b200.inputs).  The
L2 is flushed (a 256 MB write) before every timed step, outside the events.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "quantized attention TOPS (4·B·H·N²·d/t) and ms/call at N=4608 and N=34020, d=128"
DTYPE = "i8/e4m3"        # QK^T on int8 codes, PV on e4m3 codes; bf16 in and out
PRIMARY = "flux"
SECONDARIES = ("video", "long16k", "long64k")
PEAK_NOTE = "measured cuBLAS bf16 burst x 2 (nominal 8-bit/bf16 dense ratio)"
LAUNCHES_PER_STEP = 2    # k_qpass (K/V statistics, then the codes), k_attn


def _env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def _profile_traffic(record, source, workload):
    """DRAM bytes (read + written) per launch of a kernel, as counted by ncu on
    this workload (the JSON record profiles/<record>), or None when there is no
    count or the kernel's source (csrc/<source>) changed since it was taken."""
    import hashlib
    here = os.path.dirname(os.path.abspath(__file__))
    try:
        with open(os.path.join(here, "profiles", record)) as f:
            rec = json.load(f)
        with open(os.path.join(here, "quantized_attention_qk_b200", "csrc", source), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except (OSError, ValueError):
        return None
    w = rec.get("workloads", {}).get(workload)
    if rec.get("source_sha256") != sha or not w:
        return None
    return int(w["dram_bytes_read"]) + int(w["dram_bytes_write"])


def _attn_traffic(workload):
    return _profile_traffic("k_attn_traffic.txt", "sage_attn.cu", workload)


# The quantize pass's algorithmic bytes per element of B*H*N*d: Q read (2) and
# coded (1); K and V each read for their statistics (2), read again (2) and
# coded (1).
QPASS_BYTES_PER_ELEMENT = 13


def _quant_roofline(w, quant_ms, hbm_gbs, peak_kind, traffic):
    """The quantize pass against HBM bandwidth: algorithmic bytes per second
    over the measured copy bandwidth.  quant_ms runs from the step's start
    event to the event recorded before the attention kernel."""
    nbytes = QPASS_BYTES_PER_ELEMENT * w.B * w.H * w.N * w.d
    achieved = nbytes / (quant_ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": "k_qpass (statistics, then codes)", "achieved": round(achieved, 1),
            "peak": float(hbm_gbs), "unit": "GB/s", "frac": round(achieved / float(hbm_gbs), 4),
            "traffic": traffic, "algorithmic_bytes": nbytes, "quant_ms": round(quant_ms, 4),
            "peak_source": f"{peak_kind}: STREAM-style copy bandwidth"}


EX2_PER_SCORE = 0.75     # the softmax takes 2^x on the MUFU unit for 6 of every 8 scores, by polynomial for 2


def _attn_instructions(d):
    """Warp instructions per score of the dense attention kernel at head dim d,
    as counted by ncu (profiles/k_attn_instructions.txt), or None when there is
    no count or the kernel source changed since it was taken."""
    import hashlib
    here = os.path.dirname(os.path.abspath(__file__))
    try:
        with open(os.path.join(here, "profiles", "k_attn_instructions.txt")) as f:
            rec = json.load(f)
        with open(os.path.join(here, "quantized_attention_qk_b200", "csrc", "sage_attn.cu"), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except (OSError, ValueError):
        return None
    e = rec.get("head_dims", {}).get(str(d))
    if rec.get("source_sha256") != sha or not e:
        return None
    return float(e["warp_instructions"]) / float(e["scores"])


def _ex2_rate(dev):
    """Exponentials per second of the exponential unit, measured here: the
    library's ex2 probe (the softmax's own ex2.approx.ftz instruction, eight
    independent chains per thread, 8 CTAs of 256 threads per SM), 2 untimed
    and 5 timed launches, CUDA events on the current stream."""
    import torch

    import quantized_attention_qk_b200 as sage

    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    blocks, iters = 8 * sms, 2048
    sink = torch.empty(blocks * 256, dtype=torch.float32, device=dev)
    for _ in range(2):
        sage.sage_debug_ex2_probe(sink, blocks, iters)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(5):
        sage.sage_debug_ex2_probe(sink, blocks, iters)
    e1.record()
    torch.cuda.synchronize()
    return 5 * blocks * 256 * iters * 8 / (e0.elapsed_time(e1) * 1e-3)


def _softmax_roofline(w, attn_ms, kept, ex2_rate, sm_mhz, sms, instr_per_score):
    """The attention kernel against its softmax ceilings, in scores per second:
    the exponential unit (measured rate / EX2_PER_SCORE) and the issue slots
    (four warp instructions per SM and clock at the sampled SM clock, over the
    kernel's own warp instructions per score; none when there is no count for
    this source and head dim)."""
    achieved = kept * w.B * w.H * w.N * w.N / (attn_ms * 1e-3)
    ceilings = {"ex2": ex2_rate / EX2_PER_SCORE}
    if instr_per_score and sm_mhz:
        ceilings["issue"] = 4.0 * sms * sm_mhz * 1e6 / instr_per_score
    peak = min(ceilings.values())
    return {"bound": "alu", "unit": "Tscores/s", "achieved": round(achieved / 1e12, 4),
            "peak": round(peak / 1e12, 4), "frac": round(achieved / peak, 4),
            "ceilings": {k: round(v / 1e12, 4) for k, v in ceilings.items()},
            "ex2_measured_per_s": round(ex2_rate / 1e12, 4), "ex2_per_score": EX2_PER_SCORE,
            "warp_instructions_per_score": None if instr_per_score is None else round(instr_per_score, 5),
            "sm_mhz": sm_mhz}


def _workload_desc(w):
    return f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.d} {w.layout} qkv"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons of this process's GPU every
    ~2 ms (NVML, read-only queries) while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, torch_device):
        self.dev = torch_device
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.err = None
        self._stop = threading.Event()

    def start(self):
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            handle = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    handle = h
            if handle is None:
                raise RuntimeError("no NVML device matches the CUDA device")
            self.nvml, self.h = pynvml, handle
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM))
        except Exception as e:  # report, do not guess
            self.err = f"nvml unavailable: {e}"
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv, h = self.nvml, self.h
        while not self._stop.is_set():
            try:
                self.samples.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception as e:
                self.err = str(e)
                return
            time.sleep(0.002)

    def stop(self):
        self._stop.set()
        if hasattr(self, "thread"):
            self.thread.join(timeout=2)
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
               "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml, 2 ms"}
        if self.err:
            out["error"] = self.err
        return out


# --------------------------------------------------------------------------- CPU oracle baseline
def _oracle_worker(wname, cmd, results):
    """One single-threaded oracle process: on each job (seconds, seed) from
    ``cmd``, the quant emulation of random query rows of one head of the
    workload (the whole head is quantized on every call, as the oracle does)
    for about ``seconds``; None ends it."""
    os.environ["OMP_NUM_THREADS"] = "1"
    import numpy as np
    import torch

    torch.set_num_threads(1)
    import oracle
    from quantized_attention_qk_b200.inputs import WORKLOADS, make_qkv

    w = WORKLOADS[wname]
    one = w.with_(B=1, H=1, name=w.name + "-head0")
    q, k, v, _ = make_qkv(one)
    oracle.lib()
    results.put("ready")
    while True:
        job = cmd.get()
        if job is None:
            return
        seconds, seed = job
        rng = np.random.default_rng(seed)
        rows_done, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < seconds:
            rows = np.sort(rng.choice(w.N, size=32, replace=False)).astype(np.int32)
            oracle.attn_quant(q, k, v, w.sm_scale, rows=rows)
            rows_done += 32
        results.put((rows_done, time.perf_counter() - t0))


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OraclePool:
    """The CPU oracle on the host's cores: one single-threaded process per
    core (at most max_procs), each timing its own random query rows of one head
    of the workload.  The processes are spawned (not forked), so a process that
    already uses the GPU may start them."""

    def __init__(self, w, max_procs=32):
        import multiprocessing as mp

        import oracle

        oracle.build()
        self.w = w
        self.avail = host_cores()
        self.n = max(1, min(self.avail, max_procs))
        ctx = mp.get_context("spawn")
        self.cmd = [ctx.Queue() for _ in range(self.n)]
        self.res = ctx.Queue()
        self.procs = [ctx.Process(target=_oracle_worker, args=(w.name, c, self.res), daemon=True) for c in self.cmd]
        for p in self.procs:
            p.start()
        for _ in range(self.n):
            if self.res.get(timeout=600) != "ready":
                raise RuntimeError("an oracle process failed to start")

    def run(self, seconds, seed=0):
        """All processes at once for about ``seconds``.  Returns (TOPS-equivalent
        over the wall time, rows, wall seconds)."""
        t0 = time.perf_counter()
        for i, c in enumerate(self.cmd):
            c.put((seconds, seed * 1000 + i))
        got = [self.res.get(timeout=seconds + 600) for _ in range(self.n)]
        wall = time.perf_counter() - t0
        rows = sum(r for r, _ in got)
        ops = 4.0 * self.w.N * self.w.d * rows      # both contractions for the sampled rows
        return ops / wall / 1e12, rows, wall

    def close(self):
        for c in self.cmd:
            c.put(None)
        for p in self.procs:
            p.join(timeout=60)


# --------------------------------------------------------------------------- GPU arm
def run_gpu(args):
    import torch

    import quantized_attention_qk_b200 as sage
    from quantized_attention_qk_b200 import build as sage_build
    from quantized_attention_qk_b200.inputs import WORKLOADS, make_qkv
    from quantized_attention_qk_b200.replicas import Replicas, env_int, whole_job_tops

    world = env_int("WORLD_SIZE", 1)
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if not torch.cuda.is_available():
        raise SystemExit("no CUDA device")
    local = env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    reps = Replicas(device=dev)
    rank = reps.rank
    sage_build.build()
    sage.lib()
    peaks, peak_kind = _peaks()
    peak_8bit = 2.0 * float(peaks["bf16_tflops"])
    barrier = reps.barrier
    max_over_ranks = reps.max

    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def measure(w, steps, warmup):
        q, k, v, bufs = make_qkv(w, device=dev)
        out = torch.empty(w.B, w.H, w.N, w.d, dtype=torch.bfloat16, device=dev)
        sparse = args.tau is not None
        ws_fn = (sage.sage_attn_sparse_workspace_bytes if sparse else
                 sage.sage_attn_kres_workspace_bytes if args.kres else sage.sage_attn_workspace_bytes)
        ws_bytes = ws_fn(w.B, w.H, w.N, w.d)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

        def forward(events=None):
            if sparse:
                return sage.sage_attn_fwd_sparse(q, k, v, tau=args.tau, sm_scale=w.sm_scale, out=out, workspace=ws,
                                                 attn_events=events)
            if args.kres:
                return sage.sage_attn_fwd_kres(q, k, v, sm_scale=w.sm_scale, out=out, workspace=ws,
                                               attn_events=events)
            if args.fused_q:
                return sage.sage_attn_fwd_fused_q(q, k, v, sm_scale=w.sm_scale, out=out, workspace=ws,
                                                  attn_events=events)
            return sage.sage_attn_fwd(q, k, v, sm_scale=w.sm_scale, out=out, workspace=ws, attn_events=events)

        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for e in ev:
            for x in e:
                x.record()          # create the underlying events
        for _ in range(warmup):
            forward()
        torch.cuda.synchronize()
        sage.sage_check()
        barrier()
        torch.cuda.synchronize()
        clk = ClockSampler(dev)
        clk.start()
        for i in range(steps):
            flush.zero_()
            s0, a0, a1, s1 = ev[i]
            s0.record()
            forward((a0, a1))
            s1.record()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        clocks = clk.stop()
        sage.sage_check()
        step_ms = [e[0].elapsed_time(e[3]) for e in ev]
        attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
        total_ms = max_over_ranks(sum(step_ms))
        attn_avg = max_over_ranks(sum(attn_ms) / steps)
        # the kernels before the attention kernel: the quantize pass (and, when
        # selecting, the block selection)
        quant_avg = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / steps)
        kept = 1.0
        if sparse:  # fraction of (query tile, key tile) pairs the selection kept, outside the timed region
            _, mask = sage.sage_attn_fwd_sparse(q, k, v, tau=args.tau, sm_scale=w.sm_scale, out=out, workspace=ws,
                                                return_mask=True)
            kept = float(sage.mask_to_keep(mask, sage.n_tiles(w.N)).float().mean().item())
        # end to end through host memory: pinned input -> device, forward, result -> pinned host
        host_in = bufs[0].cpu().pin_memory() if w.layout == "fused" else torch.stack(bufs).cpu().pin_memory()
        ws_host = torch.empty(sage.sage_attn_fwd_host_scratch_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
        out_host = torch.empty(w.B, w.H, w.N, w.d, dtype=torch.bfloat16, pin_memory=True)
        e2e_steps = max(2, min(steps, 10))
        for _ in range(2):
            sage.sage_attn_fwd_host(host_in, w.B, w.H, w.N, w.d, layout=w.layout, sm_scale=w.sm_scale,
                                    device=dev, out_host=out_host, workspace=ws_host)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(e2e_steps):
            sage.sage_attn_fwd_host(host_in, w.B, w.H, w.N, w.d, layout=w.layout, sm_scale=w.sm_scale,
                                    device=dev, out_host=out_host, workspace=ws_host)
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps)
        sage.sage_check()
        h2d = host_in.numel() * host_in.element_size()
        d2h = out_host.numel() * out_host.element_size()
        del q, k, v, bufs, out, ws, host_in, ws_host
        torch.cuda.empty_cache()
        return dict(total_ms=total_ms, attn_ms=attn_avg, quant_ms=quant_avg, e2e_ms=e2e_ms, clocks=clocks, h2d=h2d,
                    d2h=d2h, kept=kept)

    wp = WORKLOADS[args.workload]
    r = measure(wp, args.steps, args.warmup)
    # the softmax's ceilings (outside every timed region): the exponential
    # unit measured here, the issue slots from the kernel's counted instructions
    ex2_rate = _ex2_rate(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    dense = args.tau is None and not args.kres and not args.fused_q

    def softmax_roofline(w, rr):
        return _softmax_roofline(w, rr["attn_ms"], rr["kept"], ex2_rate, rr["clocks"].get("sm_mhz"), sms,
                                 _attn_instructions(w.d) if dense else None)
    ms = r["total_ms"] / args.steps
    value = whole_job_tops(world, wp.ops, args.steps, r["total_ms"])
    attn_tops = r["kept"] * wp.ops / (r["attn_ms"] * 1e-3) / 1e12  # the kernel's own work
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": DTYPE, "data": "synthetic (seeded N(0,1) Q/K/V, K bias and outlier channels)",
        "config": {"workload": _workload_desc(wp), "B": wp.B, "H": wp.H, "N": wp.N, "d": wp.d,
                   "layout": wp.layout, "sm_scale": wp.sm_scale, "parallelism": f"replicas x{world}",
                   "l2": "flushed before every timed step (256 MB write, outside the events)"},
        "roofline": {"bound": "tensor", "kernel": "k_attn (fused attention)", "achieved": round(attn_tops, 2),
                     "peak": round(peak_8bit, 1), "unit": "TFLOP/s", "frac": round(attn_tops / peak_8bit, 4),
                     "traffic": None if (args.tau is not None or args.kres or args.fused_q) else _attn_traffic(wp.name),
                     "peak_source": f"{peak_kind}: {PEAK_NOTE}",
                     "attn_ms": round(r["attn_ms"], 4)},
        "roofline_softmax": softmax_roofline(wp, r),
        # the quantize pass of the dense forward (a selecting forward runs its
        # selection before the attention kernel too; the other modes code
        # different tensors)
        "roofline_quantize": (_quant_roofline(wp, r["quant_ms"], peaks["hbm_gbs"], peak_kind,
                                              _profile_traffic("k_qpass_traffic.txt", "sage_quant.cu", wp.name))
                              if dense else None),
        "e2e": {"value": round(world * wp.ops / (r["e2e_ms"] * 1e-3) / 1e12, 2), "unit": "TOPS",
                "ms_per_step": round(r["e2e_ms"], 4), "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "api": "sage_attn_fwd_host (pinned host qkv -> device in head chunks on three streams, quantize + "
                       "attention, bf16 out -> pinned host; dense)"},
        # a selecting forward adds the selection's scoring and ranking kernels
        # (the quantize pass pools the tiles itself)
        "gpu_launches": (LAUNCHES_PER_STEP + (2 if args.tau is not None and args.tau < 1 else 0)) * args.steps,
        "clocks": r["clocks"],
    }
    if args.tau is not None:
        line["config"]["tau"] = args.tau
        line["config"]["kept_fraction"] = round(r["kept"], 4)
        line["config"]["ops"] = ("value counts the dense 4*B*H*N^2*d; roofline.achieved counts the kept tile "
                                 "pairs only (block-sparse forward, sage_attn_fwd_sparse)")
    if args.fused_q:
        line["config"]["q_quantization"] = "in the attention kernel's prologue (sage_attn_fwd_fused_q)"
    if args.kres:
        line["config"]["k_residual"] = ("K-residual quantization (sage_attn_fwd_kres): residual codes per 64-token "
                                        "block, bf16 block means, mean term on the tensor cores")
    if args.secondary and args.workload == PRIMARY and args.tau is None and not args.kres and not args.fused_q:
        # the other full-size workloads: the video one and the long-sequence
        # sweep at 16K and 64K tokens (where the kernel's roofline is judged)
        line["secondary"] = []
        for name in SECONDARIES:
            ws_ = WORKLOADS[name]
            k2 = max(3, args.steps // 2)
            r2 = measure(ws_, k2, args.warmup)
            attn_tops2 = ws_.ops / (r2["attn_ms"] * 1e-3) / 1e12
            line["secondary"].append({
                "workload": _workload_desc(ws_), "value": round(whole_job_tops(world, ws_.ops, k2, r2["total_ms"]), 2),
                "unit": "TOPS", "ms_per_step": round(r2["total_ms"] / k2, 4), "steps": k2,
                "attn_tops": round(attn_tops2, 2), "attn_ms": round(r2["attn_ms"], 4),
                "attn_frac": round(attn_tops2 / peak_8bit, 4),
                "softmax_frac": softmax_roofline(ws_, r2)["frac"],
                "quant_ms": round(r2["quant_ms"], 4),
                "quant_frac": _quant_roofline(ws_, r2["quant_ms"], peaks["hbm_gbs"], peak_kind, None)["frac"],
                "e2e_tops": round(world * ws_.ops / (r2["e2e_ms"] * 1e-3) / 1e12, 2), "clocks": r2["clocks"]})
            line["gpu_launches"] += LAUNCHES_PER_STEP * k2
    if rank == 0 and world == 1 and args.cpu_baseline:
        pool = OraclePool(wp)
        tops, rows, secs = pool.run(args.cpu_seconds)
        pool.close()
        line["cpu_baseline"] = {"value": round(tops, 6), "unit": "TOPS", "cores": pool.n, "kind": "oracle",
                                "sample": f"{rows} query rows of one head of {wp.name} (whole-head quantization on "
                                          f"every call of 32 rows), quant-emulation mode: {pool.n} single-threaded "
                                          f"processes ({pool.avail} cores available), {secs:.1f} s wall"}
    if rank == 0:
        print(json.dumps(line, ensure_ascii=False), flush=True)
    reps.close()


# --------------------------------------------------------------------------- head-sharded arm
def run_shard(args):
    """One problem split by heads over the ranks (replicas.sharded_forward with
    the NCCL all-gather), timed on the device, the maximum over ranks."""
    import torch

    import quantized_attention_qk_b200 as sage
    from quantized_attention_qk_b200 import build as sage_build
    from quantized_attention_qk_b200.inputs import WORKLOADS, make_qkv
    from quantized_attention_qk_b200.replicas import Replicas, env_int, head_range, timed_sharded

    world = env_int("WORLD_SIZE", 1)
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if not torch.cuda.is_available():
        raise SystemExit("no CUDA device")
    local = env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    reps = Replicas(device=dev)
    sage_build.build()
    sage.lib()
    w = WORKLOADS[args.workload]
    q, k, v, bufs = make_qkv(w, device=dev)          # every rank holds the whole input
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    clk = ClockSampler(dev)
    clk.start()
    out, mine, total = timed_sharded(q, k, v, reps, args.steps, args.warmup, sm_scale=w.sm_scale,
                                     before_step=flush.zero_)
    clocks = clk.stop()
    sage.sage_check()
    # outside the timed region: the gathered result against the whole forward on this rank
    whole = sage.sage_attn_fwd(q, k, v, sm_scale=w.sm_scale)
    torch.cuda.synchronize()
    same = bool(torch.equal(out.view(torch.int16), whole.view(torch.int16)))
    same_all = reps.max(0.0 if same else 1.0) == 0.0
    h0, h1 = head_range(w.H, world, reps.rank)
    value = w.ops * args.steps / (total * 1e-3) / 1e12
    line = {"metric": METRIC, "value": round(value, 2), "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total / args.steps, 4), "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": DTYPE,
            "data": "synthetic (seeded N(0,1) Q/K/V, K bias and outlier channels)",
            "config": {"workload": _workload_desc(w), "B": w.B, "H": w.H, "N": w.N, "d": w.d, "layout": w.layout,
                       "parallelism": f"heads split over {world} GPU(s) (rank 0: heads {h0}..{h1 - 1}), "
                                      "bf16 outputs all-gathered over NCCL" + (" (no gather at one GPU)" if world == 1
                                                                              else ""),
                       "l2": "flushed before every timed step (256 MB write, outside the events)",
                       "timing": "CUDA events on each rank's stream around forward + gather; max over ranks"},
            "gathered_equals_whole_forward": same_all,
            "gpu_launches": LAUNCHES_PER_STEP * args.steps, "clocks": clocks}
    if reps.rank == 0:
        print(json.dumps(line, ensure_ascii=False), flush=True)
    del q, k, v, bufs, out, whole
    reps.close()


# --------------------------------------------------------------------------- reference arm (the CPU oracle)
def run_reference(args):
    from quantized_attention_qk_b200.inputs import WORKLOADS

    if _env_int("RANK", 0) != 0:
        return
    w = WORKLOADS[args.workload]
    per_step = max(0.5, args.cpu_seconds / max(1, args.steps))
    pool = OraclePool(w)
    for i in range(args.warmup):
        pool.run(0.2, seed=1000 + i)
    rows_total, secs_total = 0, 0.0
    for i in range(args.steps):
        _, rows, secs = pool.run(per_step, seed=i + 1)
        rows_total += rows
        secs_total += secs
    pool.close()
    value = 4.0 * w.N * w.d * rows_total / secs_total / 1e12
    sample = (f"{rows_total} query rows of one head of {w.name} over {args.steps} steps (whole-head quantization "
              f"on every call of 32 rows): {pool.n} single-threaded oracle processes ({pool.avail} cores "
              f"available), {secs_total:.1f} s wall")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs_total / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (fp32 quant steps)",
            "data": "synthetic", "config": {"workload": _workload_desc(w), "B": w.B, "H": w.H, "N": w.N, "d": w.d},
            "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": pool.n, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line, ensure_ascii=False), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["sage", "reference"], default="sage")
    ap.add_argument("--workload", default=PRIMARY)
    ap.add_argument("--no-secondary", dest="secondary", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--tau", type=float, default=None,
                    help="time the block-sparse forward with this tau instead of the dense one")
    ap.add_argument("--kres", action="store_true",
                    help="time the K-residual forward instead of the smoothing one")
    ap.add_argument("--fused-q", dest="fused_q", action="store_true",
                    help="time the forward that quantizes Q in the attention kernel's prologue")
    ap.add_argument("--shard", action="store_true",
                    help="split one problem by heads over the GPUs and all-gather the outputs (strong scaling)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.shard:
        run_shard(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the Muir chunkwise gated delta rule on B200 GPUs.

One step = the whole hot path over one batch of the long-context workload
(B=1, H=16, T=32768, dk=dv=128, chunk 128, bf16 inputs): ``muir_chunk_fwd``
(saving chunk states) followed by ``muir_chunk_bwd`` with a random upstream
gradient.  The streaming-decode step (B=64, H=16, d=128, float32 state) is
measured in the same run and reported under ``"decode"``, the q/k feature
prologue (forward and backward) under ``"qk_prologue"``.

Usage::

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl muir|reference]

N > 1 runs one process per GPU (launched by torch.distributed.run; started as
a single process, the script relaunches itself that way); every rank
processes its own batch (weak scaling, no data-path collective); the time is
the max over ranks.  ``--impl reference`` times the fp64 CPU oracle on a
bounded sample of the same workload (rank 0 only).  Prints ONE JSON line.
"""
from __future__ import annotations

import argparse
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WID = 2
METRIC = "Muir chunk fwd+bwd tokens/s & % bf16 TC peak (H=16,d=128,T=32K); decode GB/s"
NAMES = ["q", "k", "v", "g", "e", "w", "gamma"]

# Nominal dense tensor-core ratios (TF32 : BF16 = 1.1 : 2.25 PFLOP/s per GPU).
TF32_OVER_BF16 = 1.1 / 2.25


def flops_fwd_per_token_head(C: int, d: int) -> float:
    """Algorithmic forward FLOPs per token and head (2 per multiply-add,
    triangular products counted at half size): 9Cd + C^2/3 + 8d^2."""
    return 9 * C * d + C * C / 3 + 8 * d * d


# Algorithmic HBM bytes per token and head (bf16 I/O, one pass, nothing saved):
BYTES_FWD = 7 * 256 + 256            # 7 inputs read, o written
BYTES_BWD = 8 * 256 + 7 * 256        # 7 inputs + dO read, 7 gradients written
DECODE_BYTES_PER_HEAD = 2 * 128 * 128 * 4 + 6 * 128 * 2 + 128 * 2  # S read+write, tokens, o

# DRAM traffic per launch from ncu (dram__bytes_read.sum + dram__bytes_write.sum),
# keyed by kernel; valid only while the chunk-kernel source hash matches.
NCU_TRAFFIC = {
    # ncu --set full of one k2_bwd2 launch at B=1 H=16 T=8192 (131,072 token-heads):
    # 476.6 MB read + 154.5 MB written; traffic scales with the chunks processed
    "k2_bwd2": {"bytes_per_token_head": (476.6144e6 + 154.4576e6) / 131072,
                "source": "3028ae8d4b2a9580"},
}


CHUNK_KERNEL_FILES = ("chunk", "fwd2.cu", "bwd2.cu")


def source_hash(chunk_kernels_only: bool = False) -> str:
    """Hash of the library sources; with ``chunk_kernels_only`` of the files the
    chunk kernels are compiled from (``chunk*.cu``, ``fwd2.cu``, ``bwd2.cu`` and
    every header), so that counters taken on those kernels stay valid across
    changes elsewhere and are dropped when those kernels change."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_115_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if chunk_kernels_only and not (f.startswith(CHUNK_KERNEL_FILES) or f.endswith((".cuh", ".h"))):
            continue
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["muir", "reference"], default="muir")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="target CPU time of the oracle sample")
    p.add_argument("--T", type=int, default=None,
                   help="shorter sequence for profiling captures (not a bench number)")
    a = p.parse_args(argv)
    if a.warmup < 3:
        p.error("--warmup must be >= 3")
    if a.steps < 1:
        p.error("--steps must be >= 1")
    return a


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a float over all ranks (identity when world == 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Seed of this rank's batch: rank 0 draws the canonical workload."""
    return 1000 + WID + 7919 * rank


def rank_batch(rank: int, **over):
    """This rank's batch of the workload (CPU tensors): every rank draws its
    own inputs from its own seed (weak scaling: no data is exchanged)."""
    from gated_delta_rule_115_b200 import inputs as I
    return I.chunk_inputs(WID, seed=rank_seed(rank), **over)


def timed_steps(step, steps: int, warmup: int, world: int, timer, barrier=None,
                device=None) -> float:
    """The timing protocol of every arm: ``warmup`` untimed steps, a barrier,
    exactly ``steps`` timed steps, a barrier; returns ms per step, the max over
    ranks.  ``timer()`` returns ``(start, stop)`` callables, stop() giving the
    elapsed ms (CUDA events on the launching stream for the GPU arm)."""
    for _ in range(warmup):
        step()
    if barrier is not None:
        barrier()
    start, stop = timer()
    start()
    for _ in range(steps):
        step()
    ms = stop()
    if barrier is not None:
        barrier()
    return max_over_ranks(ms, world, device) / steps


def job_tokens_per_s(ms_per_step: float, tokens_per_rank: int, world: int) -> float:
    """Whole-job throughput: the tokens all ranks processed per step over the
    slowest rank's step time."""
    return tokens_per_rank * world / (ms_per_step / 1e3)


def spawn_command(args_list, gpus: int, port: int):
    """The command that runs this script once per GPU (one process per GPU,
    rendezvous on 127.0.0.1), forwarding the script's own arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={gpus}", "--master-addr", "127.0.0.1", "--master-port", str(port),
            os.path.abspath(__file__)] + list(args_list)


# ------------------------------------------------------------------ clocks

CLOCK_FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
                "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
                "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]


class ClockSampler:
    """nvidia-smi sampling every 200 ms while the timed region runs."""

    def __init__(self, gpu_id: str):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        cmd = ["nvidia-smi", "--query-gpu=" + ",".join(CLOCK_FIELDS), "--format=csv,noheader,nounits",
               "-lms", "200"]
        if gpu_id:
            cmd += ["-i", gpu_id]
        try:
            self.p = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self) -> dict:
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.strip().split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        self.f.close()
        os.unlink(self.f.name)
        out = summarize_clocks(rows)
        out["sampler"] = "nvidia-smi, 200 ms"
        return out


class NvmlClockSampler:
    """In-process NVML reads every ``period`` seconds on a background thread
    while the timed region runs, so that a region of a few hundred
    milliseconds still gets several samples.  Only queries: no clock, limit or
    mode of the GPU is changed.  Rows take the nvidia-smi sampler's form."""

    # NVML clock-event reason bits, in the order summarize_clocks reads them
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, gpu_id: str, nvml=None, period: float = 0.01):
        if nvml is None:
            import pynvml as nvml
        self.nvml = nvml
        nvml.nvmlInit()
        try:
            self.h = (nvml.nvmlDeviceGetHandleByUUID(gpu_id) if gpu_id
                      else nvml.nvmlDeviceGetHandleByIndex(0))
            self.max_mhz = nvml.nvmlDeviceGetMaxClockInfo(self.h, nvml.NVML_CLOCK_SM)
            self.reasons = (getattr(nvml, "nvmlDeviceGetCurrentClocksEventReasons", None)
                            or nvml.nvmlDeviceGetCurrentClocksThrottleReasons)
            self.rows = []
            self._sample()  # a query that fails, fails here rather than in the thread
        except Exception:
            nvml.nvmlShutdown()
            raise
        self.rows = []  # (that sample precedes the region)
        self.period = period
        self.done = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _sample(self):
        n = self.nvml
        sm = n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM)
        watts = n.nvmlDeviceGetPowerUsage(self.h) / 1000.0
        mask = int(self.reasons(self.h))
        flags = ["Active" if mask & bit else "Not Active" for _, bit in self.REASONS]
        self.rows.append([str(sm), str(self.max_mhz), "%.1f" % watts, hex(mask)] + flags)

    def _run(self):
        while not self.done.wait(self.period):
            try:
                self._sample()
            except Exception:
                return

    def stop(self) -> dict:
        self.done.set()
        self.thread.join(timeout=5)
        try:
            self.nvml.nvmlShutdown()
        except Exception:
            pass
        out = summarize_clocks(list(self.rows))
        out["sampler"] = "nvml, %d ms" % round(self.period * 1e3)
        return out


def clock_sampler(gpu_id: str):
    """The NVML sampler, or nvidia-smi's where NVML cannot be read."""
    try:
        return NvmlClockSampler(gpu_id)
    except Exception:
        return ClockSampler(gpu_id)


def summarize_clocks(rows) -> dict:
    sm, mx, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for r in rows:
        r = [x.strip() for x in r]
        if len(r) < 8:
            continue
        try:
            sm.append(float(r[0]))
            mx.append(float(r[1]))
        except ValueError:
            continue
        for n, v in zip(names, r[4:8]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
            "samples": len(sm)}


# ------------------------------------------------------------------ oracle arm

def oracle_tokens(T_s: int, threads: int) -> float:
    """Seconds the fp64 oracle (token-loop forward + BPTT backward) takes on
    all 16 heads of the first T_s tokens of the workload."""
    import oracle
    from gated_delta_rule_115_b200 import inputs as I
    oracle.build()
    x = I.chunk_inputs(WID, T=T_s)
    t0 = time.perf_counter()
    oracle.fwd(*[x[n] for n in NAMES], S0=x["S0"], threads=threads)
    oracle.bwd(*[x[n] for n in NAMES], S0=x["S0"], dO=x["dO"], ckpt=128, threads=threads)
    return time.perf_counter() - t0


def oracle_sample_size(seconds: float, threads: int) -> int:
    """Tokens T_s (multiple of 128, <= 32768) whose oracle run takes about `seconds`."""
    t_cal = oracle_tokens(128, threads)
    return int(max(128, min(32768, 128 * seconds / max(t_cal, 1e-3))) // 128 * 128)


def sample_desc(T_s: int) -> str:
    return f"fwd+bwd of B=1, all H=16 heads, first T={T_s} tokens of the workload (tokens/s = T_s / seconds)"


def oracle_sample(seconds: float, threads: int):
    T_s = oracle_sample_size(seconds, threads)
    dt = oracle_tokens(T_s, threads)
    return T_s / dt, sample_desc(T_s), dt


def reference_arm(args, rank, world):
    """The oracle as the reference arm: each step is one bounded sample of the
    workload, sized so that warm-up plus timed steps take about two minutes."""
    if rank != 0:
        return None
    threads = len(os.sched_getaffinity(0))
    per = max(0.5, 120.0 / (args.steps + args.warmup))
    T_s = oracle_sample_size(per, threads)
    times = []
    for i in range(args.warmup + args.steps):
        dt = oracle_tokens(T_s, threads)
        if i >= args.warmup:
            times.append(dt)
    dt = statistics.median(times)
    value = T_s / dt
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample_desc(T_s)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def workload_config(T=32768):
    return {"workload": f"long-context chunkwise fwd+bwd, B=1 H=16 T={T} dk=dv=128 chunk=128",
            "B": 1, "H": 16, "T": T, "d": 128, "chunk": 128, "io_dtype": "bf16",
            "l2": "per-step inputs (0.94 GB) and outputs exceed the 126 MB L2; no extra flush"}


# ------------------------------------------------------------------ GPU arm

def gpu_arm(args, rank, world, local):
    import torch
    import gated_delta_rule_115_b200 as muir
    from gated_delta_rule_115_b200 import inputs as I
    from gated_delta_rule_115_b200 import build as B
    B.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    L = muir.lib()
    W = I.WORKLOADS[WID]
    if args.T is not None:
        import dataclasses
        W = dataclasses.replace(W, T=args.T)
    x = rank_batch(rank, T=W.T)
    d = {k: (v.to(dev) if v is not None else None) for k, v in x.items()}
    C = W.chunk
    args_in = [d[n] for n in NAMES]

    def step():
        o, S, Sc, Mc, aux = muir.chunk_fwd(*args_in, d["S0"], chunk=C, return_saved=True,
                                           save_aux=True, ws=ws_f)
        gr = muir.chunk_bwd(*args_in, d["S0"], d["dO"], chunk=C, S_chunks=Sc, M_chunks=Mc,
                            aux=aux, ws=ws_b)
        return o, gr

    ws_f = torch.empty(muir.fwd_workspace_bytes(W.B, W.T, W.H, W.dk, C), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(muir.bwd_workspace_bytes(W.B, W.T, W.H, W.dk, C), dtype=torch.uint8, device=dev)
    gpu_id = ""
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    st = torch.cuda.current_stream(dev)
    sampler = None

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    def timer():
        nonlocal sampler
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def start():
            nonlocal sampler
            sampler = clock_sampler(gpu_id)
            L.muir_profile_reset()
            L.muir_profile_enable(1)
            e0.record(st)

        def stop():
            e1.record(st)
            torch.cuda.synchronize()
            L.muir_profile_enable(0)
            return e0.elapsed_time(e1)
        return start, stop

    ms = timed_steps(step, args.steps, args.warmup, world, timer, barrier, dev)
    L.muir_profile_collect()
    clocks = sampler.stop()
    prof = {L.muir_profile_name(i).decode(): (L.muir_profile_total_ms(i), L.muir_profile_launches(i))
            for i in range(L.muir_profile_count())}
    launches = sum(n for _, n in prof.values())
    value = job_tokens_per_s(ms, W.B * W.T, world)
    token_heads = W.B * W.T * W.H
    fl = 3 * flops_fwd_per_token_head(C, W.dk) * token_heads * world
    tflops = fl / (ms / 1e3) / 1e12

    peaks = load_peaks()
    # dominant kernel
    dom = max(prof.items(), key=lambda kv: kv[1][0])
    dom_name, (dom_ms, dom_n) = dom
    dom_avg = dom_ms / max(dom_n, 1)
    roof = kernel_roofline(dom_name, dom_avg, token_heads, C, W.dk, peaks)

    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16+fp16+tf32",
        "data": "synthetic", "config": workload_config(W.T),
        "tflops": tflops, "tc_peak_frac": tflops / peaks["bf16_tflops"],
        "hbm_gbs_algorithmic": (BYTES_FWD + BYTES_BWD) * token_heads * world / (ms / 1e3) / 1e9,
        "roofline": roof,
        "kernels_ms_per_step": {k: v[0] / args.steps for k, v in sorted(prof.items())},
        "gpu_launches": launches,
        "clocks": clocks,
        "source": source_hash(),
        "chunk_kernel_source": source_hash(chunk_kernels_only=True),
    }
    if not args.no_e2e:
        out["e2e"] = e2e_measure(muir, x, W, C, dev, ws_f, ws_b, args.steps, world)
    if not args.no_decode:
        out["decode"] = decode_measure(muir, I, dev, peaks)
        out["qk_prologue"] = qk_measure(muir, dev, peaks)
        out["other_workloads"] = configs_measure(muir, I, dev, peaks)
        out["fused_stages"] = fused_measure(muir, I, dev, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = len(os.sched_getaffinity(0))
        v, desc, dt = oracle_sample(args.cpu_seconds, threads)
        out["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                               "sample": desc, "seconds": dt}
    return out


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def kernel_work(name, C, d):
    """Algorithmic (bytes, flops) per token-head credited to one launch of a
    chunk kernel: each product counted once at 2 flops per multiply-add, the
    decay-masked and triangular ones at half size; bytes = the bf16 inputs the
    kernel reads and the outputs it writes (saved intermediates excluded)."""
    F = flops_fwd_per_token_head(C, d)
    return {
        # 8 decay-masked gradient products and the 4 dL matrices they use
        "k2_bwd2": (11 * 256, 12 * C * d),
        # Y, dY, dYR, dU and the four state-side products
        "k2_bwd1": (10 * 256, 4 * C * d + 14 * d * d),
        # masked products, inverse, solve, Z and the chunk transition
        "k2_intra": (7 * 256, 10 * C * d + C * C / 3 + 6 * d * d),
        "k2_chain": (2 * d * d * 4 / C, 2 * d * d * d / C),
        "k2_chain_rev": (2 * d * d * 4 / C, 2 * d * d * d / C),
        "k2_out": (256, 2 * d * d),
    }.get(name, (BYTES_FWD, F))


def kernel_roofline(name, avg_ms, token_heads, C, d, peaks):
    """Roofline of one launch of the dominant kernel from its algorithmic work.
    The tensor peak is TF32 (sustained bf16 x 1.1/2.25): the kernels mix TF32
    products with 16-bit ones, so TF32 is the lower of the two ceilings."""
    work = kernel_work(name, C, d)
    byts = work[0] * token_heads
    fl = work[1] * token_heads
    gbs = byts / (avg_ms / 1e3) / 1e9
    tfl = fl / (avg_ms / 1e3) / 1e12
    tf32_peak = peaks["bf16_tflops_sustained"] * TF32_OVER_BF16
    f_hbm, f_tc = gbs / peaks["hbm_gbs"], tfl / tf32_peak
    traffic = None
    t = NCU_TRAFFIC.get(name)
    if t and t.get("source") == source_hash(chunk_kernels_only=True):
        traffic = t["bytes_per_token_head"] * token_heads
    if f_hbm >= f_tc:
        r = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": f_hbm}
    else:
        r = {"bound": "tensor", "achieved": tfl, "peak": tf32_peak, "unit": "TFLOP/s", "frac": f_tc}
    r.update({"traffic": traffic, "kernel": name, "avg_launch_ms": avg_ms,
              "peak_source": peaks["source"] + (" (tf32 = sustained bf16 x 1.1/2.25)" if r["bound"] == "tensor" else ""),
              "other_bound_frac": f_tc if r["bound"] == "hbm" else f_hbm})
    return r


def e2e_measure(muir, x, W, C, dev, ws_f, ws_b, steps, world):
    """The same step through the public API with host buffers: per step, copy
    the inputs from pinned host memory, run forward + backward, copy o and all
    gradients back to pinned host memory.  As an input pipeline does, the
    copies run on their own streams and overlap the compute of neighbouring
    steps: inputs are double-buffered on the device (step i+2's copy waits for
    step i's compute), and step i's results are read back while step i+1
    computes.  The timed region runs from before step 1's first input copy to
    after step K's last result copy; every step's copies are inside it."""
    import torch
    host = {k: v.pin_memory() for k, v in x.items() if v is not None}
    slots = [{k: torch.empty_like(v, device=dev) for k, v in host.items()} for _ in range(2)]
    outs_host = None
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = 0

    def run(n, e0=None):
        nonlocal outs_host, d2h
        in_done = [torch.cuda.Event() for _ in range(n)]
        cmp_done = [torch.cuda.Event() for _ in range(n)]
        if e0 is not None:
            e0.record(s_in)
        for i in range(n):
            slot = slots[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(cmp_done[i - 2])
                for k, v in host.items():
                    slot[k].copy_(v, non_blocking=True)
                in_done[i].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(in_done[i])
                a = [slot[nm] for nm in NAMES]
                o, S, Sc, Mc, aux = muir.chunk_fwd(*a, slot.get("S0"), chunk=C, return_saved=True,
                                                   save_aux=True, ws=ws_f)
                gr = muir.chunk_bwd(*a, slot.get("S0"), slot["dO"], chunk=C, S_chunks=Sc,
                                    M_chunks=Mc, aux=aux, ws=ws_b)
                res = [o, S] + [gr[k] for k in sorted(gr)]
                cmp_done[i].record(s_cmp)
            if outs_host is None:
                outs_host = [torch.empty_like(r, device="cpu").pin_memory() for r in res]
                d2h = sum(r.numel() * r.element_size() for r in res)
            with torch.cuda.stream(s_out):
                s_out.wait_event(cmp_done[i])
                for hbuf, r in zip(outs_host, res):
                    hbuf.copy_(r, non_blocking=True)
                    r.record_stream(s_out)  # keep r alive until its copy is done

    torch.cuda.synchronize()
    run(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(steps, e0)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world, dev)
    return {"value": W.B * W.T * world / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
            "steps": steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "overlap": "input copies, compute and result copies on three streams, "
                       "double-buffered device inputs"}


def decode_measure(muir, I, dev, peaks, steps=50):
    """Decode step (B=64, H=16, d=128, float32 state, static gamma): each timed
    step is bracketed by CUDA events with a 256 MB L2 flush in between, so the
    state really comes from HBM.  Also reports CUDA-graph replay of 1,000
    back-to-back steps (state resident in L2)."""
    import torch
    W = I.WORKLOADS[4]
    S0, gstat = I.decode_state()
    S = S0.to(dev)
    tok = {k: v.to(dev) for k, v in I.decode_tokens(0).items()}
    gam = gstat.to(dev)
    o = torch.empty(W.B, W.H, W.dv, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream(dev)

    def one():
        muir.recurrent_step(tok["q"], tok["k"], tok["v"], tok["g"], tok["e"], tok["w"], gam, S,
                            gamma_static=True, o=o)

    for _ in range(5):
        one()
    times = []
    for _ in range(steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        one()
        b.record(st)
        b.synchronize()
        times.append(a.elapsed_time(b))
    ms = statistics.median(times)
    byts = DECODE_BYTES_PER_HEAD * W.B * W.H
    gbs = byts / (ms / 1e3) / 1e9
    # graph replay, L2 resident
    g = torch.cuda.CUDAGraph()
    s2 = torch.cuda.Stream(dev)
    s2.wait_stream(st)
    with torch.cuda.stream(s2):
        one()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s2):
            for _ in range(100):
                one()
    st.wait_stream(s2)
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(10):
        g.replay()
    b.record(st)
    torch.cuda.synchronize()
    ms_g = a.elapsed_time(b) / 1000
    # a batch whose state (1 GiB) is far beyond the 126 MB L2: back-to-back
    # steps read and write it from HBM without any flush
    BL = 1024
    S_l, g_l = I.decode_state(B=BL)
    S_l = S_l.to(dev)
    tok_l = {k: v.to(dev) for k, v in I.decode_tokens(0, B=BL).items()}
    g_l = g_l.to(dev)
    o_l = torch.empty(BL, W.H, W.dv, dtype=torch.bfloat16, device=dev)

    def one_l():
        muir.recurrent_step(tok_l["q"], tok_l["k"], tok_l["v"], tok_l["g"], tok_l["e"],
                            tok_l["w"], g_l, S_l, gamma_static=True, o=o_l)

    for _ in range(5):
        one_l()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(steps):
        one_l()
    b.record(st)
    torch.cuda.synchronize()
    ms_l = a.elapsed_time(b) / steps
    byts_l = DECODE_BYTES_PER_HEAD * BL * W.H
    large = {"B": BL, "H": W.H, "state_bytes": BL * W.H * 128 * 128 * 4, "ms_per_step": ms_l,
             "gbs": byts_l / (ms_l / 1e3) / 1e9,
             "hbm_frac": byts_l / (ms_l / 1e3) / 1e9 / peaks["hbm_gbs"],
             "tokens_per_s": BL / (ms_l / 1e3),
             "note": "state 1 GiB >> L2: consecutive steps stream it from HBM, no flush"}
    del S_l, tok_l, o_l
    return {
        "workload": "decode step B=64 H=16 d=128, fp32 state, bf16 tokens, static gamma",
        "large_batch": large,
        "ms_per_step_l2_flushed": ms, "gbs_l2_flushed": gbs,
        "hbm_frac": gbs / peaks["hbm_gbs"], "tokens_per_s": W.B / (ms / 1e3),
        "bytes_per_step": byts,
        "graph_replay_ms_per_step": ms_g, "graph_replay_gbs_l2_resident": byts / (ms_g / 1e3) / 1e9,
        "note": "graph replay keeps the 64 MiB state in L2; the flushed number is the HBM one",
    }


def configs_measure(muir, I, dev, peaks, steps=5, warmup=3):
    """The other chunked workloads, each timed with CUDA events over ``steps``
    back-to-back calls after ``warmup`` (inputs far beyond L2):
    the layer-shaped forward (B=8, H=16, T=4096, d=128, its chunk 64, and
    chunk 128, the on-chip path) and the large-chunk stress workload's
    forward+backward (B=2, H=8, T=8192, chunk 256, the 8-token panel path for
    its large decay spans, and chunk 128)."""
    import torch
    st = torch.cuda.current_stream(dev)

    def timeit(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for _ in range(steps):
            fn()
        b.record(st)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps

    out = {}
    W1 = I.WORKLOADS[1]
    x = I.chunk_inputs(1)
    d = {k: (v.to(dev) if v is not None else None) for k, v in x.items()}
    del x
    th = W1.B * W1.T * W1.H
    for C in (W1.chunk, 128):
        ws = torch.empty(muir.fwd_workspace_bytes(W1.B, W1.T, W1.H, W1.dk, C), dtype=torch.uint8,
                         device=dev)
        ms = timeit(lambda: muir.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=C, ws=ws))
        out[f"layer_fwd_chunk{C}"] = {
            "workload": f"layer-shaped forward B={W1.B} H={W1.H} T={W1.T} d={W1.dk} chunk {C}, bf16",
            "ms": ms, "tokens_per_s": W1.B * W1.T / (ms / 1e3),
            "gbs_algorithmic": BYTES_FWD * th / (ms / 1e3) / 1e9,
            "hbm_frac": BYTES_FWD * th / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}
        del ws
    del d
    W3 = I.WORKLOADS[3]
    x = I.chunk_inputs(3, with_dO=True)
    d = {k: (v.to(dev) if v is not None else None) for k, v in x.items()}
    del x
    for C in (W3.chunk, 128):
        wf = torch.empty(muir.fwd_workspace_bytes(W3.B, W3.T, W3.H, W3.dk, C), dtype=torch.uint8,
                         device=dev)
        wb = torch.empty(muir.bwd_workspace_bytes(W3.B, W3.T, W3.H, W3.dk, C), dtype=torch.uint8,
                         device=dev)

        def fb():
            _, _, Sc, Mc, aux = muir.chunk_fwd(*[d[n] for n in NAMES], d["S0"], chunk=C,
                                               return_saved=True, save_aux=True, ws=wf)
            muir.chunk_bwd(*[d[n] for n in NAMES], d["S0"], d["dO"], chunk=C, S_chunks=Sc,
                           M_chunks=Mc, aux=aux, ws=wb)
        ms = timeit(fb)
        out[f"stress_fwd_bwd_chunk{C}"] = {
            "workload": f"large-chunk stress fwd+bwd B={W3.B} H={W3.H} T={W3.T} d={W3.dk} chunk {C}, bf16",
            "ms": ms, "tokens_per_s": W3.B * W3.T / (ms / 1e3)}
        del wf, wb
    return out


def fused_measure(muir, I, dev, peaks, steps=5, warmup=3):
    """The long-context step with every fused stage on: raw q and k (the
    SiLU + L2-norm prologue inside the chunk kernels) and the five gate
    families projected from one latent row per token (R = 512, ranks 64, 64,
    128, 128, 128; the output gate applied in the output epilogue).  Gate
    inputs per token-head: the latent shared by the 16 heads (1,024 B / 16)
    instead of four gate tensors (4 x 256 B)."""
    import torch
    W = I.WORKLOADS[WID]
    x = I.fused_inputs(WID, with_dO=True)
    lat, proj = I.gate_latent_inputs(W.B, W.T, W.H)
    d = {k: (v.to(dev) if v is not None else None) for k, v in x.items()}
    latd = lat.to(dev)
    projd = {f: (off, U.to(dev), b.to(dev)) for f, (off, U, b) in proj.items()}
    del x, lat
    st = torch.cuda.current_stream(dev)

    def step():
        o, S, sv = muir.chunk_fwd_fused(d["xq"], d["xk"], d["v"], None, None, None, None, d["S0"],
                                        qk_raw=True, latent=latd, proj=projd)
        return muir.chunk_bwd_fused(d["xq"], d["xk"], d["v"], None, None, None, None, d["S0"],
                                    d["dO"], qk_raw=True, saved=sv, latent=latd, proj=projd)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(steps):
        step()
    b.record(st)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    R = sum(I.GATE_RANKS.values())
    return {"workload": f"long-context fwd+bwd B={W.B} H={W.H} T={W.T} d=128 chunk 128, raw q/k, "
                        f"gates projected from a latent of R={R}",
            "ms": ms, "tokens_per_s": W.B * W.T / (ms / 1e3),
            "gate_input_bytes_per_token_head": R * 2 / W.H,
            "gate_input_bytes_per_token_head_unfused": 4 * 128 * 2}


def qk_measure(muir, dev, peaks, steps=20):
    """q/k prologue (SiLU + unit L2 norm per row, forward and backward) over
    the long-context workload's q and k: 2 x 524,288 rows of 128 bf16.  Each
    timed call moves 268 MB (forward: read + write) or 403 MB (backward: x and
    dy read, dx written), beyond the 126 MB L2, with a 256 MB flush between
    calls.  GB/s from those algorithmic bytes."""
    import torch
    g = torch.Generator(device=dev).manual_seed(11)
    x = torch.randn(2, 32768, 16, 128, generator=g, device=dev).to(torch.bfloat16)
    dy = torch.randn(2, 32768, 16, 128, generator=g, device=dev).to(torch.bfloat16)
    y, dx = torch.empty_like(x), torch.empty_like(x)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream(dev)
    nbytes = x.numel() * 2

    def timed(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            fn()
            b.record(st)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    ms_f = timed(lambda: muir.qk_prologue(x, out=y))
    ms_b = timed(lambda: muir.qk_prologue_bwd(x, dy, out=dx))
    gf = 2 * nbytes / (ms_f / 1e3) / 1e9
    gb = 3 * nbytes / (ms_b / 1e3) / 1e9
    return {
        "workload": "q and k of B=1 H=16 T=32768 d=128, bf16 (1,048,576 rows)",
        "fwd_ms": ms_f, "fwd_gbs": gf, "fwd_hbm_frac": gf / peaks["hbm_gbs"],
        "bwd_ms": ms_b, "bwd_gbs": gb, "bwd_hbm_frac": gb / peaks["hbm_gbs"],
    }


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # started as one process: run one rank per GPU under torch.distributed.run
        import socket
        sk = socket.socket()
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
        sk.close()
        argv_list = sys.argv[1:] if argv is None else list(argv)
        return subprocess.call(spawn_command(argv_list, args.gpus, port))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if args.impl == "reference":
        out = reference_arm(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return 0
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    try:
        out = gpu_arm(args, rank, world, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

#!/usr/bin/env python
"""Benchmark of the hot path: one 5-step Newton-Schulz msign of a 4096 x 4096
bf16 matrix (Jordan's coefficients), reported as ms per msign call and
useful TFLOP/s against the measured dense BF16 tensor-core peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One process per GPU (torchrun for N > 1).  Every rank runs its own msign
calls on its own matrix (the problems are independent: weak scaling, no
collective on the data path); the step time is the max over ranks.

Timing: W untimed warm-up calls, then K timed calls.  Before each timed call
an L2 flush writes a 256 MiB buffer (larger than the 126 MB L2); each call is
bracketed by CUDA events on the launching stream and the K durations are
summed.  The library's launch records are on during those K calls (CUDA
events around every kernel, on the same stream), so the roofline of the
dominant kernel and the launch count come from the timed calls themselves; a
second pass without the records reports what they cost.

The reference arm (--impl reference) times the fp64 CPU oracle on the host
cores, rank 0 only, on a bounded sample of the same workload.
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

METRIC = "ms per msign call and useful TFLOP/s (% of B200 dense BF16 peak), 4096² bf16"
N_ROWS = N_COLS = 4096
T_STEPS = 5
FLUSH_BYTES = 256 << 20

# dram__bytes_read.sum + dram__bytes_write.sum of the one gemm_sm100_kernel
# launch (all 15 products, chained) of a 4096^2 msign call, from the ncu
# capture summarised in profiles/gemm_sm100_msign4096.md; valid only for the
# kernel source whose hash is recorded with it.
NCU_TRAFFIC = {"bytes_per_launch": 1186.81e6, "kernel_sha": "293a2f59ad5eb25a"}


def useful_flops(n: int, m: int, steps: int) -> float:
    """Triangle-counted useful FLOPs of one NS call on an oriented n x m matrix:
    per step X X^T (m n (n+1)), A A (n^2 (n+1)) and B X (2 n^2 m)."""
    return float(steps * (m * n * (n + 1) + n * n * (n + 1) + 2 * n * n * m))


def kernel_sha() -> str:
    h = hashlib.sha256()
    for f in ("gemm_sm100.cuh", "ptx_sm100.cuh"):
        with open(os.path.join(ROOT, "newton_schulz_msign_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"bf16_tflops": d.get("bf16_tflops"), "bf16_tflops_sustained": d.get("bf16_tflops_sustained"),
                "hbm_gbs": d.get("hbm_gbs"), "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


# ---------------------------------------------------------------- ranks

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(world: int, backend: str = "nccl"):
    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity on one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ---------------------------------------------------------------- clocks

def wait_idle(event) -> None:
    """Waits for `event` by polling with sleeps, which release the GIL so the
    clock sampler keeps sampling while the GPU works."""
    import torch

    while not event.query():
        time.sleep(0.0005)
    torch.cuda.synchronize()


class ClockSampler:
    """Polls NVML (read-only) every 5 ms: SM clock, max SM clock, power and
    the active clock-event reasons, for the duration of the timed region."""

    REASONS = {
        "hw_slowdown": 0x0000000000000008,
        "hw_thermal_slowdown": 0x0000000000000040,
        "hw_power_brake_slowdown": 0x0000000000000080,
        "sw_thermal_slowdown": 0x0000000000000020,
        "sw_power_cap": 0x0000000000000004,
    }

    def __init__(self, index: int):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: report no clocks rather than fail the run
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                power = nv.nvmlDeviceGetPowerUsage(self._h) / 1000.0
                self.samples.append((mhz, reasons, power))
            except Exception:
                pass
            time.sleep(0.005)

    def start(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self) -> dict:
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        reasons = sorted({name for _, r, _ in self.samples for name, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples), "power_w_max": max(s[2] for s in self.samples)}


# ---------------------------------------------------------------- CPU oracle

def time_oracle(target_s: float = 20.0):
    """Times the fp64 oracle's msign on the host.  Runs 4096^2 itself when a
    1024^2 probe predicts it fits in ~target_s, else the largest power-of-two
    size that does, scaled by the FLOP ratio.  Returns (ms per 4096^2 call,
    cores, sample description)."""
    import numpy as np

    from oracle import ns_oracle as O

    try:
        from threadpoolctl import threadpool_info

        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count() or 1])
    except Exception:
        cores = os.cpu_count() or 1

    def run(n):
        x = np.random.default_rng(0).standard_normal((n, n)).astype(np.float32)
        t0 = time.perf_counter()
        O.msign_ns(x, input_cast="bf16")
        return time.perf_counter() - t0

    n = 1024
    t = run(n)
    while n < N_ROWS and t * 8 < target_s:
        n *= 2
        t = run(n)
    scale = useful_flops(N_ROWS, N_COLS, T_STEPS) / useful_flops(n, n, T_STEPS)
    desc = (f"one {n}x{n} fp64 NS msign (5 steps) on the host"
            + ("" if n == N_ROWS else f", scaled x{scale:.0f} by the FLOP ratio to 4096^2"))
    return t * scale * 1e3, cores, desc, t


# ---------------------------------------------------------------- our arm

def run_ours(args):
    import numpy as np
    import torch

    import newton_schulz_msign_b200 as msb
    from newton_schulz_msign_b200 import synth

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init(world)
    stream = torch.cuda.current_stream()

    x = synth.momentum_like_torch(N_ROWS, N_COLS, seed=1000 + rank, device=dev).to(torch.bfloat16).contiguous()
    out = torch.empty_like(x)
    ws = torch.empty(msb.msign_ns_workspace_size(1, N_ROWS, N_COLS), dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    for _ in range(args.warmup):
        msb.msign_ns(x, out, workspace=ws)
    msb.sync_status()

    def timed_pass(instrumented: bool):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        msb.profile_reset()
        msb.profile_enable(instrumented)
        barrier(world)
        torch.cuda.synchronize()
        for k in range(args.steps):
            flush.fill_(k & 0xFF)
            ev[k][0].record(stream)
            msb.msign_ns(x, out, workspace=ws)
            ev[k][1].record(stream)
        wait_idle(ev[-1][1])
        barrier(world)
        msb.profile_enable(False)
        msb.sync_status()
        return [a.elapsed_time(b) for a, b in ev]

    # the headline: K calls, each between two events, with the library's
    # launch records on (CUDA events around every kernel, on the same stream),
    # so that the roofline of the dominant kernel comes from the same calls
    clocks = ClockSampler(local)
    clocks.start()
    per_call = timed_pass(True)
    clk = clocks.stop()
    total_ms = sum(per_call)
    kinds = {k: msb.profile_read(k) for k in ("gemm", "norm", "ingest", "elementwise")}
    msb.profile_reset()
    # the same K calls again without launch records: what the records cost
    per_call_plain = timed_pass(False)

    # end to end through the public call with host buffers (msign_ns_host:
    # the copy of the pinned input in, the iteration and the copy of the
    # result out, all on the call's stream), calls alternating between two
    # streams so that one call's copies overlap the other's kernels, as a
    # pipelined caller runs them; the whole run between two events on the
    # current stream.  No L2 flush here: each call's device data (the input
    # copied in, ~190 MB of intermediates) exceeds the 126 MB L2, and a flush
    # kernel queued behind the other stream's GEMM would hold back this
    # stream's copy
    host_in = [x.cpu().pin_memory() for _ in range(2)]
    host_out = [torch.empty_like(host_in[0]).pin_memory() for _ in range(2)]
    e2e_need = msb.msign_ns_host_workspace_size(1, N_ROWS, N_COLS)
    e2e_ws = [torch.empty(e2e_need, dtype=torch.uint8, device=dev) for _ in range(2)]
    e2e_streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]

    def e2e_run(steps):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for s in e2e_streams:
            s.wait_event(start)
        for k in range(steps):
            s = e2e_streams[k % 2]
            msb.msign_ns_host(host_in[k % 2], host_out[k % 2], workspace=e2e_ws[k % 2], stream=s)
        for s in e2e_streams:
            done = torch.cuda.Event()
            done.record(s)
            stream.wait_event(done)
        end.record(stream)
        torch.cuda.synchronize()
        return start.elapsed_time(end)

    e2e_run(2)
    barrier(world)
    torch.cuda.synchronize()
    e2e_ms = e2e_run(args.steps)
    barrier(world)
    msb.sync_status()

    max_total = max_over_ranks(total_ms, world, dev)
    max_e2e = max_over_ranks(e2e_ms, world, dev)
    units = world * args.steps
    ms_per_call = max_total / units
    e2e_per_call = max_e2e / units
    flops = useful_flops(N_ROWS, N_COLS, T_STEPS)
    tflops = flops * units / (max_total / 1e3) / 1e12

    peaks = measured_peaks()
    g = kinds["gemm"]
    achieved = g["flops"] / (g["ms"] / 1e3) / 1e12 if g["ms"] > 0 else None
    traffic = NCU_TRAFFIC["bytes_per_launch"] if NCU_TRAFFIC["kernel_sha"] == kernel_sha() else None
    roofline = {
        "bound": "tensor", "kernel": "gemm_sm100_kernel", "achieved": achieved, "peak": peaks["bf16_tflops"],
        "unit": "TFLOP/s", "frac": (achieved / peaks["bf16_tflops"]) if achieved else None, "traffic": traffic,
        "peak_source": f"{peaks['source']} bf16 burst",
        # K back-to-back calls hold the GPU at its power cap (see clocks):
        # the same figure against the sustained cuBLAS loop
        "peak_sustained": peaks["bf16_tflops_sustained"],
        "frac_sustained": (achieved / peaks["bf16_tflops_sustained"])
        if achieved and peaks["bf16_tflops_sustained"] else None,
        "launches": g["launches"], "avg_launch_ms": g["ms"] / max(g["launches"], 1),
        "flops_per_launch": g["flops"] / max(g["launches"], 1),
        "share_of_call_time": g["ms"] / total_ms if total_ms > 0 else None,
        "measured": "launch records (CUDA events around every library launch) of the K timed calls themselves",
    }
    launches = sum(v["launches"] for v in kinds.values())  # of the K timed calls

    result = {
        "metric": METRIC, "value": ms_per_call, "unit": "ms/call", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_call * world, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "msign_ns 4096x4096 bf16, 5-step quintic NS, Jordan (3.4445, -4.7750, 2.0315)",
                   "rows": N_ROWS, "cols": N_COLS, "ns_steps": T_STEPS, "batch_per_gpu": 1,
                   "input": "momentum-like U diag(i^-0.8) V^T + N(0,1e-3^2) noise, seed 1000+rank",
                   "l2": "flushed (256 MiB write) before every timed call", "parallelism": f"replicas x{world}"},
        "useful_tflops": tflops, "frac_of_peak": tflops / peaks["bf16_tflops"],
        "frac_of_sustained_peak": tflops / peaks["bf16_tflops_sustained"] if peaks["bf16_tflops_sustained"] else None,
        "useful_flops_per_call": flops,
        "roofline": roofline,
        "e2e": {"value": e2e_per_call, "unit": "ms/call", "h2d_bytes_per_step": host_in[0].numel() * 2,
                "d2h_bytes_per_step": host_out[0].numel() * 2, "api": "msign_ns_host (C ABI, host buffers)",
                "streams": 2, "timed": "whole run between two events, calls pipelined over the two streams",
                "l2": "not flushed: each call's device data (input copied in, intermediates) exceeds L2"},
        "gpu_launches": launches,
        "clocks": clk,
        "other_kernels": {k: {"launches": v["launches"], "ms": v["ms"], "bytes": v["bytes"]}
                          for k, v in kinds.items() if k != "gemm"},
        "per_call_ms": {"min": min(per_call), "median": statistics.median(per_call), "max": max(per_call),
                        "without_launch_records_median": statistics.median(per_call_plain)},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ms, cores, desc, secs = time_oracle()
        result["cpu_baseline"] = {"value": ms, "unit": "ms/call", "cores": cores, "kind": "oracle", "sample": desc,
                                  "sample_seconds": secs}
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# ---------------------------------------------------------------- other workloads
#
# `--workload NAME` times one of the other configurations the tests cover,
# with the same rules as the headline (warm-up, L2 flush before each timed
# call, CUDA events on the launching stream, clocks sampled meanwhile).
# Useful FLOPs come from the library's own launch records (triangle-counted
# per product), so they match the headline's bookkeeping.  These lines are
# measurements for the record beside the headline metric.

WORKLOADS = {
    # the single-matrix case: 256 x 512 fp32 N(0,1) input, bf16 compute (latency-bound)
    "msign_256x512": ("msign", dict(batch=1, rows=256, cols=512, io="fp32", gaussian=True)),
    "msign_8x4096": ("msign", dict(batch=8, rows=4096, cols=4096)),
    "msign_4x4096x11008": ("msign", dict(batch=4, rows=4096, cols=11008)),
    "msign_2048": ("msign", dict(batch=1, rows=2048, cols=2048)),
    "msign_1024x4096": ("msign", dict(batch=1, rows=1024, cols=4096)),
    "msign_4096_fp32": ("msign", dict(batch=1, rows=4096, cols=4096, compute="fp32")),
    "msign_4096_improved_init": ("msign", dict(batch=1, rows=4096, cols=4096, improved=True)),
    # the headline call with its phases as separate launches (msign_set_chaining(0)),
    # for per-phase timing and profiles of X X^T, the A^2 product and B X
    "msign_4096_phases": ("msign", dict(batch=1, rows=4096, cols=4096, chaining=False)),
    "gram_xxt_1024": ("gram_xxt", dict(n=1024)),
    "gram_xxt_2048": ("gram_xxt", dict(n=2048)),
    "gram_xxt_4096": ("gram_xxt", dict(n=4096)),
    "gram_xxt_8192": ("gram_xxt", dict(n=8192)),
    "gram_ns_1024x4096": ("gram_ns", dict(rows=1024, cols=4096)),
    "gram_ns_1024x16384": ("gram_ns", dict(rows=1024, cols=16384)),
    "gram_ns_2048x4096": ("gram_ns", dict(rows=2048, cols=4096)),
    "gram_ns_2048x16384": ("gram_ns", dict(rows=2048, cols=16384)),
    # the same wide shapes through standard NS, for the Gram-NS comparison
    "msign_1024x16384": ("msign", dict(batch=1, rows=1024, cols=16384)),
    "msign_2048x4096": ("msign", dict(batch=1, rows=2048, cols=4096)),
    "msign_2048x16384": ("msign", dict(batch=1, rows=2048, cols=16384)),
    "muon_llama3_8b_layer": ("muon", dict()),
    # the automatic route (Gram NS where msign_ns_route picks it)
    "msign_4x4096x11008_auto": ("msign", dict(batch=4, rows=4096, cols=11008, method="auto")),
    "msign_1024x16384_auto": ("msign", dict(batch=1, rows=1024, cols=16384, method="auto")),
    "muon_llama3_8b_layer_auto": ("muon", dict(method="auto")),
    # the whole 32-layer stack (224 matrices), G redrawn before every step
    "muon_llama3_8b_stack": ("muon", dict(layers=32)),
    "muon_llama3_8b_stack_auto": ("muon", dict(layers=32, method="auto")),
    # Mousse: the per-step direction given the factor roots, and the roots
    "mousse_direction_4096": ("mousse", dict(n=4096)),
    "mousse_inv_root_4096": ("mousse_root", dict(n=4096, iters=20)),
}


def run_workload(args):
    import torch

    import newton_schulz_msign_b200 as msb
    from newton_schulz_msign_b200 import synth

    kind, cfg = WORKLOADS[args.workload]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    desc = {"workload": args.workload}
    redraw = None  # per-step input refresh outside the timed region
    if kind == "msign":
        b, r, c = cfg["batch"], cfg["rows"], cfg["cols"]
        comp = cfg.get("compute", "bf16")
        if cfg.get("gaussian"):
            x = torch.from_numpy(synth.gaussian((b, r, c), seed=0)).to(dev)
        else:
            x = torch.stack([synth.momentum_like_torch(r, c, seed=2000 + i, device=dev) for i in range(b)])
        x = x.to({"bf16": torch.bfloat16, "fp32": torch.float32}[cfg.get("io", "bf16")]).contiguous()
        out = torch.empty_like(x)
        ws = torch.empty(msb.msign_ns_workspace_size(b, r, c, comp), dtype=torch.uint8, device=dev)
        imp = cfg.get("improved", False)
        meth = cfg.get("method", "standard")
        call = lambda: msb.msign_ns(x, out, compute=comp, improved_init=imp, method=meth, workspace=ws)
        if not cfg.get("chaining", True):
            msb.set_chaining(False)
            desc.update(chaining="one launch per product")
        desc.update(batch=b, rows=r, cols=c, compute=comp,
                    input=("N(0,1) seed 0, " if cfg.get("gaussian") else "momentum-like, ") + cfg.get("io", "bf16"),
                    improved_init=imp, method=meth,
                    route=msb.msign_ns_route(b, r, c, comp, method=meth, improved_init=imp))
    elif kind == "gram_xxt":
        n = cfg["n"]
        x = synth.gaussian_torch((n, n), seed=3000, device=dev, std=1.0 / n ** 0.5, dtype=torch.bfloat16)
        a = torch.empty(n, n, dtype=torch.bfloat16, device=dev)
        call = lambda: msb.gram_xxt(x, a)
        desc.update(n=n, m=n, input="N(0, 1/m) bf16", output="full n x n bf16, exactly symmetric")
    elif kind == "gram_ns":
        r, c = cfg["rows"], cfg["cols"]
        x = synth.gaussian_torch((r, c), seed=4000, device=dev, dtype=torch.bfloat16)
        out = torch.empty_like(x)
        ws = torch.empty(msb.gram_ns_workspace_size(1, r, c), dtype=torch.uint8, device=dev)
        call = lambda: msb.gram_ns(x, out, workspace=ws)
        desc.update(rows=r, cols=c, input="N(0,1) bf16", inner="fp16", restart_after=[2])
    elif kind == "mousse":
        n = cfg["n"]
        gen = torch.Generator(device=dev)
        gen.manual_seed(7000)
        Gs = [torch.randn(n, n, generator=gen, device=dev) * 1e-2 for _ in range(2)]
        Lf = sum(G_ @ G_.T for G_ in Gs)
        Rf = sum(G_.T @ G_ for G_ in Gs)
        eps = float(1e-3 * torch.trace(Lf) / n)
        Lr = msb.mousse_inv_root(Lf[None], eps=eps, iters=22)
        Rr = msb.mousse_inv_root(Rf[None], eps=eps, iters=22)
        del Gs, Lf, Rf
        g = synth.momentum_like_torch(n, n, seed=7001, device=dev).to(torch.bfloat16)[None].contiguous()
        out = torch.empty_like(g)
        ws = torch.empty(msb._lib.lib().mousse_direction_workspace_size(1, n, n), dtype=torch.uint8, device=dev)
        call = lambda: msb.mousse_direction(g, Lr, Rr, out, workspace=ws)
        desc.update(rows=n, cols=n, input="momentum-like bf16 G; L, R = sums of two Gaussian G G^T, G^T G, "
                    "damped by 1e-3 of their mean eigenvalue; roots from mousse_inv_root",
                    note="per step: L^-1/4 msign(L^-1/4 G R^-1/4) R^-1/4 with the roots given")
    elif kind == "mousse_root":
        n, iters = cfg["n"], cfg["iters"]
        gen = torch.Generator(device=dev)
        gen.manual_seed(7000)
        Gs = [torch.randn(n, n, generator=gen, device=dev) * 1e-2 for _ in range(2)]
        Lf = sum(G_ @ G_.T for G_ in Gs)[None].contiguous()
        eps = float(1e-3 * torch.trace(Lf[0]) / n)
        del Gs
        out = torch.empty_like(Lf)
        ws = torch.empty(msb._lib.lib().mousse_inv_root_workspace_size(1, n), dtype=torch.uint8, device=dev)
        call = lambda: msb.mousse_inv_root(Lf, out, eps=eps, iters=iters, workspace=ws)
        desc.update(n=n, iters=iters, compute="fp32-accurate (3xTF32)",
                    input="L = sum of two Gaussian G G^T, damped by 1e-3 of its mean eigenvalue")
    else:
        layers = cfg.get("layers", 1)
        shapes = [(r, c) for _ in range(layers) for _, r, c in synth.llama3_8b_layer_shapes()]
        W = [synth.gaussian_torch(s_, seed=5000 + i, device=dev, std=0.02, dtype=torch.bfloat16)
             for i, s_ in enumerate(shapes)]
        M = [torch.zeros(s_, dtype=torch.float32, device=dev) for s_ in shapes]
        G = [synth.gaussian_torch(s_, seed=6000 + i, device=dev, std=1e-4, dtype=torch.bfloat16)
             for i, s_ in enumerate(shapes)]
        ws = torch.empty(msb.muon_step_workspace_size(shapes), dtype=torch.uint8, device=dev)
        meth = cfg.get("method", "standard")
        call = lambda: msb.muon_step(W, M, G, momentum=0.95, lr=0.02, method=meth, workspace=ws)
        if layers > 1:
            gen = torch.Generator(device=dev)
            gen.manual_seed(6999)

            def redraw():  # a fresh gradient for every step, drawn before the step's timing starts
                for g_ in G:
                    g_.normal_(0.0, 1e-4, generator=gen)
        desc.update(matrices=[list(s_) for s_ in shapes[:7]], layers=layers, w="bf16", m="fp32",
                    g="N(0, 1e-4^2) bf16" + (", redrawn before every step" if layers > 1 else ""),
                    momentum=0.95, lr=0.02, method=meth, workspace_bytes=ws.numel(),
                    note=f"{layers} Llama-3-8B decoder layer(s) of 7 matrices; every call is a further step")
    for _ in range(args.warmup):
        call()
    msb.sync_status()

    def timed(instrumented):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        msb.profile_reset()
        msb.profile_enable(instrumented)
        torch.cuda.synchronize()
        for k in range(args.steps):
            if redraw is not None:
                redraw()
            flush.fill_(k & 0xFF)
            ev[k][0].record(stream)
            call()
            ev[k][1].record(stream)
        wait_idle(ev[-1][1])
        msb.profile_enable(False)
        msb.sync_status()
        return [a_.elapsed_time(b_) for a_, b_ in ev]

    clocks = ClockSampler(0)
    clocks.start()
    per_call = timed(False)
    clk = clocks.stop()
    timed(True)
    kinds = {k: msb.profile_read(k) for k in ("gemm", "norm", "ingest", "elementwise")}
    msb.profile_reset()
    ms = statistics.median(per_call)
    g = kinds["gemm"]
    fp32 = cfg.get("compute", "bf16") == "fp32" or kind == "mousse_root"
    # the launch records count the fp32-accurate path's three tf32 passes
    flops = g["flops"] / args.steps / (3.0 if fp32 else 1.0)
    peaks = measured_peaks()
    pk = peaks["bf16_tflops"] * (0.5 if fp32 else 1.0)  # tf32 runs at half the bf16 rate
    achieved = g["flops"] / (g["ms"] / 1e3) / 1e12 if g["ms"] > 0 else None
    # useful FLOPs: those of the products that ran (Gram NS's on its route)
    print(json.dumps({
        "workload": args.workload, "metric": "ms per call and useful TFLOP/s", "value": ms, "unit": "ms/call",
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": False,
        "per_call_ms": {"min": min(per_call), "median": ms, "max": max(per_call)},
        "useful_flops_per_call": flops, "useful_tflops": flops / (ms / 1e3) / 1e12,
        "frac_of_peak": flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
        "roofline": {"bound": "tensor", "kernel": "gemm_sm100_kernel", "achieved": achieved, "peak": pk,
                     "unit": "TFLOP/s", "frac": achieved / pk if achieved else None,
                     "launches_per_call": g["launches"] / args.steps,
                     "peak_source": peaks["source"] + (" bf16 burst" if pk == peaks["bf16_tflops"] else
                                                       " bf16 burst x 1/2 (tf32 rate)")},
        "gpu_launches_per_call": sum(v["launches"] for v in kinds.values()) / args.steps,
        "other_kernels": {k: {"launches": v["launches"], "ms": v["ms"]} for k, v in kinds.items() if k != "gemm"},
        "clocks": clk, "config": desc, "l2": "flushed (256 MiB write) before every timed call", "data": "synthetic",
    }), flush=True)


# ---------------------------------------------------------------- reference arm

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import numpy as np

    from oracle import ns_oracle as O

    try:
        from threadpoolctl import threadpool_info

        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count() or 1])
    except Exception:
        cores = os.cpu_count() or 1
    # each step: one bounded sample of the workload, an n x n fp64 NS msign,
    # with n chosen so the whole run stays within a few minutes
    budget_s = 150.0
    n = 512
    x = np.random.default_rng(0).standard_normal((n, n)).astype(np.float32)
    t0 = time.perf_counter()
    O.msign_ns(x, input_cast="bf16")
    t = time.perf_counter() - t0
    while n < N_ROWS and t * 8 * (args.steps + args.warmup) < budget_s:
        n *= 2
        x = np.random.default_rng(0).standard_normal((n, n)).astype(np.float32)
        t0 = time.perf_counter()
        O.msign_ns(x, input_cast="bf16")
        t = time.perf_counter() - t0
    x = np.random.default_rng(0).standard_normal((n, n)).astype(np.float32)
    for _ in range(args.warmup):
        O.msign_ns(x, input_cast="bf16")
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        O.msign_ns(x, input_cast="bf16")
        times.append(time.perf_counter() - t0)
    scale = useful_flops(N_ROWS, N_COLS, T_STEPS) / useful_flops(n, n, T_STEPS)
    ms = sum(times) / len(times) * scale * 1e3
    sample = (f"one {n}x{n} fp64 NS msign per step on {cores} host threads"
              + ("" if n == N_ROWS else f", scaled x{scale:.0f} by the FLOP ratio to 4096^2"))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": ms, "unit": "ms/call", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "msign_ns 4096x4096, 5-step quintic NS, Jordan (3.4445, -4.7750, 2.0315)",
                   "rows": N_ROWS, "cols": N_COLS, "ns_steps": T_STEPS, "parallelism": "host cores"},
        "cpu_baseline": {"value": ms, "unit": "ms/call", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": ms, "unit": "ms/call", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the host oracle timing")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=None,
                    help="time another configuration instead of the headline (1 GPU)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.workload is not None:
        run_workload(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

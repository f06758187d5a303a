"""Benchmark of the B200 attention core on the 336 px ViT-L/14 batch.

Workload: B=256 images, N=577 tokens (576 patches + CLS), H=16 heads, d=64,
packed bf16 QKV drawn by the seeded generator (synthetic data of the encoder's
shape).  One step = one call of the fused attention kernel over the whole
batch.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  python bench.py --configs     # per-config report (one JSON line per item, 1 GPU)
  python bench.py --block       # LayerNorm / linear layers, whole encoder layers and encoders
  python bench.py --linear M,K,N   # one linear layer of that shape
  python bench.py --layer WORKLOAD # one encoder layer, stage by stage

Under torchrun every rank runs the same per-GPU batch on its own GPU (weak
scaling, no collective on the data path); the elapsed time is the max over
ranks.  ``--impl reference`` times the fp64 CPU oracle on the host cores on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import glob
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import seeded_inputs as si  # noqa: E402

WORKLOAD = si.VIT_L14_336PX_B256
METRIC = "attention TFLOP/s (4*B*H*N^2*d per call) on B200"
UNIT = "TFLOP/s"
# Device code of the attention kernel: an ncu summary describes the current kernel
# only while these files are unchanged (host-side edits do not invalidate it).
KERNEL_SOURCES = ["vit_self_attention_b200/csrc/attn_kernel.cuh",
                  "vit_self_attention_b200/csrc/ptx.cuh"]


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0,
            "source": "fallback"}


def ncu_summary(workload: str) -> tuple[dict, str | None]:
    """Figures of the committed ncu summary of this kernel and workload, if it was taken
    on the current kernel sources: ``dram_bytes_per_full_launch`` (DRAM bytes read +
    written by one launch) and ``tensor_pipe_active_pct`` (sm__pipe_tensor_cycles_active,
    percent of peak); ({}, None) when there is none."""
    cur = kernel_source_hash()
    found: dict = {}
    src = None
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        with open(path) as f:
            txt = f.read()
        m_w = re.search(r"^workload:\s*(\S+)", txt, re.M)
        m_h = re.search(r"^kernel_source_sha256_16:\s*([0-9a-f]+)", txt, re.M)
        if not (m_w and m_h and m_w.group(1) == workload and m_h.group(1) == cur):
            continue
        for key in ("dram_bytes_per_full_launch", "tensor_pipe_active_pct"):
            m = re.search(rf"^{key}:\s*([0-9.eE+]+)", txt, re.M)
            if m and key not in found:
                found[key] = float(m.group(1))
                src = os.path.relpath(path, ROOT) if src is None else src
    return found, src


def ncu_traffic(workload: str) -> tuple[float | None, str | None]:
    """DRAM bytes per launch from the committed ncu summary of this kernel and workload,
    if it was taken on the current kernel sources (else None)."""
    found, src = ncu_summary(workload)
    if "dram_bytes_per_full_launch" not in found:
        return None, None
    return found["dram_bytes_per_full_launch"], src


_REASON_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML from before the warm-up to the
    end of the timed region; the summary keeps the samples taken inside the timed region
    (host times t0..t1 set by mark_start / mark_end)."""

    def __init__(self, device_index: int, period_s: float = 0.0002):
        self.samples: list[tuple[float, int, int]] = []
        self._t0 = None
        self._t1 = None
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = int(pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM))
            self._ok = True
        except Exception:  # NVML missing: report no clocks
            self._ok = False
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                t = time.perf_counter()
                mhz = int(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                reasons = int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
                self.samples.append((t, mhz, reasons))
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._ok:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._ok:
            self._t.join()

    def mark_start(self):
        self._t0 = time.perf_counter()

    def mark_end(self):
        self._t1 = time.perf_counter()

    def summary(self) -> dict | None:
        if not self._ok or not self.samples:
            return None
        t0 = self._t0 if self._t0 is not None else float("-inf")
        t1 = self._t1 if self._t1 is not None else float("inf")
        inside = [(m, r) for t, m, r in self.samples if t0 <= t <= t1]
        if not inside:  # a region shorter than one NVML query: the last sample before it
            before = [(m, r) for t, m, r in self.samples if t < t0]
            inside = before[-1:]
        if not inside:
            return None
        mhz = [m for m, _ in inside]
        seen = 0
        for _, r in inside:
            seen |= r
        names = sorted(n for bit, n in _REASON_BITS.items() if seen & bit and n != "gpu_idle")
        return {"sm_mhz": float(statistics.median(mhz)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(mhz), "sm_mhz_min": min(mhz),
                "sm_mhz_max_seen": max(mhz)}


# ---------------------------------------------------------------- oracle (CPU)
def cpu_oracle_rate(target_s: float, max_heads: int | None = None) -> dict:
    """Time the fp64 oracle on whole (b, h) heads of the workload, doubling the sample
    until one run takes at least target_s; returns TFLOP/s of the last run."""
    import oracle
    c = WORKLOAD
    threads = oracle.default_threads()
    images = 1
    bits_cache = {}
    last = None
    while True:
        if images not in bits_cache:
            bits_cache.clear()
            bits_cache[images] = si.packed_qkv(images, c.N, c.H, c.d, c.seed(0))
        bits = bits_cache[images]
        t0 = time.perf_counter()
        oracle.attention_packed_bf16(bits, c.scale, threads=threads)
        dt = time.perf_counter() - t0
        flops = 4.0 * images * c.H * c.N * c.N * c.d
        last = {"value": flops / dt / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
                "sample": f"{images} image(s) x {c.H} heads of the B=256 N=577 H=16 d=64 batch "
                          f"({images * c.H} of {c.B * c.H} heads), fp64, {dt:.2f} s",
                "seconds": dt}
        if dt >= target_s or images >= c.B or (max_heads and images * c.H >= max_heads):
            return last
        images = min(c.B, images * 2 if dt < target_s / 4 else images + max(1, images // 2))


def run_reference(args, rank: int, world: int) -> None:
    if rank != 0:
        return
    c = WORKLOAD
    import oracle
    threads = oracle.default_threads()
    # Size one step so warm-up + timed steps end within about two minutes.
    per_step = max(0.5, min(5.0, 120.0 / max(1, args.steps + args.warmup)))
    probe = cpu_oracle_rate(0.2)
    heads_per_s = probe["value"] * 1e12 / (4.0 * c.N * c.N * c.d)
    images = int(max(1, min(c.B, round(per_step * heads_per_s / c.H))))
    bits = si.packed_qkv(images, c.N, c.H, c.d, c.seed(0))
    for _ in range(args.warmup):
        oracle.attention_packed_bf16(bits, c.scale, threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.attention_packed_bf16(bits, c.scale, threads=threads)
    dt = time.perf_counter() - t0
    flops = 4.0 * images * c.H * c.N * c.N * c.d * args.steps
    value = flops / dt / 1e12
    sample = (f"each step: {images} image(s) x {c.H} heads of the B=256 N=577 H=16 d=64 batch, "
              f"fp64 oracle on {threads} host threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded splitmix64 Box-Muller, bf16)",
        "config": {"workload": c.name, "B": c.B, "N": c.N, "H": c.H, "d": c.d,
                   "images_per_step": images},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "images_per_s_24_layers": value * 1e12 / (4.0 * c.H * c.N * c.N * c.d) / 24.0,
    }
    print(json.dumps(line), flush=True)


def max_over_ranks(values, world: int, device=None):
    """Element-wise max of per-rank timings over all ranks (identity on one rank)."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def rank_seed(rank: int) -> int:
    """Seed of a rank's batch: every rank draws its own images (weak scaling)."""
    return WORKLOAD.seed(0) + 7919 * rank


# ---------------------------------------------------------------- CUDA path
def run_ours(args, rank: int, world: int, local_rank: int) -> None:
    import torch
    import torch.distributed as dist

    import vit_self_attention_b200 as vab

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    c = WORKLOAD
    if args.images is not None:
        c = dataclasses.replace(c, B=int(args.images), name=f"{c.name}_B{int(args.images)}")
    stream = torch.cuda.current_stream(dev)

    bits = si.packed_qkv(c.B, c.N, c.H, c.d, rank_seed(rank))
    host_in = torch.from_numpy(bits.view(np.int16)).pin_memory()
    qkv = host_in.to(dev, non_blocking=False).view(torch.bfloat16)
    out = torch.empty((c.B, c.N, c.H, c.d), dtype=torch.bfloat16, device=dev)
    base = qkv.data_ptr()
    step_b = c.H * c.d * 2

    def step():
        vab.vla_attn_fwd(base, base + step_b, base + 2 * step_b, out, c.B, c.N, c.H, c.d,
                         c.scale, stream)

    def barrier():
        if world > 1:
            dist.barrier()

    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        for _ in range(max(3, args.warmup)):
            step()
        torch.cuda.synchronize()
        launches0 = vab.vla_attn_launch_count()
        barrier()
        torch.cuda.synchronize()
        clocks.mark_start()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        clocks.mark_end()
        barrier()
    launches = vab.vla_attn_launch_count() - launches0
    ms = ev0.elapsed_time(ev1)
    st, site = vab.vla_attn_last_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status {st} (site {site}) after the timed region")

    # ---- end-to-end through the host-buffer C-ABI entry (pinned host memory)
    e2e_steps = max(2, min(args.steps, 10))
    e2e_ms = float("nan")
    if not args.no_e2e:
        host_out = torch.empty((c.B, c.N, c.H, c.d), dtype=torch.int16).pin_memory()
        dev_in = torch.empty(bits.shape, dtype=torch.int16, device=dev)
        dev_out = torch.empty((c.B, c.N, c.H, c.d), dtype=torch.int16, device=dev)

        def e2e_step():
            vab.vla_attn_fwd_host(host_in, host_out, dev_in, dev_out, c.B, c.N, c.H, c.d,
                                  c.scale, stream)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = e0.elapsed_time(e1)

    ms, e2e_ms = max_over_ranks([ms, e2e_ms], world, dev)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_oracle_rate(args.cpu_seconds)
        cpu = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
    if rank != 0:
        return
    line = build_line(c, world, args.steps, max(3, args.warmup), ms,
                      None if args.no_e2e else (e2e_ms, e2e_steps, int(bits.nbytes)),
                      int(launches), clocks.summary(), cpu)
    print(json.dumps(line), flush=True)


def build_line(c, world: int, steps: int, warmup: int, ms: float, e2e, launches: int,
               clocks: dict | None, cpu: dict | None) -> dict:
    """The bench's JSON line from the max-over-ranks timings: ``ms`` for ``steps`` device
    steps of one ``c.B``-image batch per rank, ``e2e`` = (ms, steps, input bytes per step)
    of the host-buffer leg or None."""
    flops_call = float(c.flops())
    ms_step = ms / steps
    value = flops_call * world * steps / (ms / 1e3) / 1e12
    peaks = measured_peaks()
    achieved = flops_call / (ms_step / 1e3) / 1e12
    prof, prof_src = ncu_summary(c.name)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded splitmix64 Box-Muller, bf16)",
        "config": {"workload": c.name, "B": c.B, "N": c.N, "H": c.H, "d": c.d,
                   "scale": c.scale, "flops_per_call": c.flops(),
                   "hbm_bytes_per_call": c.bytes(),
                   "l2": "inputs larger than L2 (1.21 GB of QKV + O per step vs 126 MB L2)"},
        "images_per_s_24_layers": world * c.B / (ms_step / 1e3) / 24.0,
        "roofline": {"bound": "tensor", "achieved": achieved,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"],
                     "traffic": prof.get("dram_bytes_per_full_launch"),
                     "peak_source": f"{peaks['source']} bf16 burst (cuBLAS)",
                     "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                     "hbm_gbs_achieved": c.bytes() / (ms_step / 1e3) / 1e9,
                     "hbm_frac": c.bytes() / (ms_step / 1e3) / 1e9 / peaks["hbm_gbs"],
                     "tensor_pipe_active_pct": prof.get("tensor_pipe_active_pct"),
                     "ncu_source": prof_src},
        "cpu_baseline": cpu,
        "e2e": None,
        "gpu_launches": int(launches),
        "clocks": clocks,
        "kernel_source_sha256_16": kernel_source_hash(),
    }
    if e2e is not None:
        e2e_ms, e2e_steps, in_bytes = e2e
        line["e2e"] = {
            "value": flops_call * world * e2e_steps / (e2e_ms / 1e3) / 1e12, "unit": UNIT,
            "h2d_bytes_per_step": int(in_bytes),
            "d2h_bytes_per_step": int(c.B * c.N * c.H * c.d * 2),
            "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
            "api": "vla_attn_fwd_host (pinned host buffers)"}
    return line


def _percentile(xs, q):
    xs = sorted(xs)
    return xs[min(len(xs) - 1, int(round(q * (len(xs) - 1))))]


def run_configs(args) -> None:
    """Per-config report on one GPU: warm (back-to-back calls in a CUDA graph) and
    cold-L2 (after a 256 MB write) per-call time (median, P95)
    and roofline fraction for every workload, the L-layer sequence replayed from one
    CUDA graph with fresh buffers per layer (configs 1-4), longer sequences
    (384 px and 448 px ViT-L/14 grids), and the fp64 oracle on all host cores and
    on one core."""
    import torch

    import oracle
    import vit_self_attention_b200 as vab

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = measured_peaks()
    p_bf16 = float(peaks.get("bf16_tflops", 1590.0)) * 1e12
    hbm = float(peaks.get("hbm_gbs", 6650.0)) * 1e9
    scratch = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > L2 (126 MB)

    def buffers(c, bits):
        qkv = torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)
        out = torch.empty((c.B, c.N, c.H, c.d), dtype=torch.bfloat16, device=dev)
        return qkv, out

    def call(c, qkv, out):
        b = qkv.data_ptr()
        st = c.H * c.d * 2
        vab.vla_attn_fwd(b, b + st, b + 2 * st, out, c.B, c.N, c.H, c.d, c.scale)

    def timed(c, qkv, out, iters, flush):
        ts = []
        for i in range(iters):
            if flush:
                scratch.fill_(i & 0xFF)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            call(c, qkv, out)
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)  # us
        return ts

    items = [(c, True) for c in si.WORKLOADS] + [
        (si.AttnConfig(6, "vit_l14_384px_b64", 64, 730, 16, 64, 0.125, 1.0, 1.0, 1, 24), False),
        (si.AttnConfig(7, "vit_l14_448px_b64", 64, 1025, 16, 64, 0.125, 1.0, 1.0, 1, 24), False)]
    for c, std in items:
        bits = c.qkv(0) if std else si.packed_qkv(c.B, c.N, c.H, c.d, 4242 + c.N)
        qkv, out = buffers(c, bits)
        for _ in range(10):
            call(c, qkv, out)
        torch.cuda.synchronize()
        iters = 20 if c.B * c.N >= 100000 else 100
        # Warm: 20 back-to-back calls on the same buffers in one CUDA graph, so the
        # host-side cost of a call (argument checks, tensor-map encoding) does not
        # leave the GPU idle between calls; per-call time = replay time / 20.
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            call(c, qkv, out)
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize()
        g20 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g20, stream=side):
            for _ in range(20):
                call(c, qkv, out)
        for _ in range(3):
            g20.replay()
        torch.cuda.synchronize()
        warm = []
        for _ in range(max(5, iters // 20)):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            g20.replay()
            e1.record()
            e1.synchronize()
            warm.append(e0.elapsed_time(e1) * 1e3 / 20)
        del g20
        # Eager: 200 calls enqueued back to back from Python (argument checks, cached
        # tensor maps, launch); the host enqueue time per call and the wall time per
        # call until the stream drains (host-bound when the first is the larger).
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(200):
            call(c, qkv, out)
        t1 = time.perf_counter()
        torch.cuda.synchronize()
        t2 = time.perf_counter()
        eager = {"host_enqueue_us": (t1 - t0) / 200 * 1e6, "wall_us": (t2 - t0) / 200 * 1e6}
        # Cold L2: a 256 MB write before each call; the call is enqueued while that
        # write runs, so the events bracket the kernel alone.
        cold = timed(c, qkv, out, min(iters, 50), True)
        flops, nbytes = c.flops(), c.bytes()
        t_roof = max(flops / p_bf16, nbytes / hbm) * 1e6
        rec = {"mode": "configs", "workload": c.name, "B": c.B, "N": c.N, "H": c.H, "d": c.d,
               "bound": "tensor" if flops / p_bf16 > nbytes / hbm else "hbm",
               "roofline_us": t_roof,
               "warm_us": {"median": statistics.median(warm), "p95": _percentile(warm, 0.95)},
               "cold_l2_us": {"median": statistics.median(cold), "p95": _percentile(cold, 0.95)},
               "eager_us": eager,
               "tflops_warm": flops / statistics.median(warm) / 1e6,
               "frac_warm": t_roof / statistics.median(warm),
               "frac_cold_l2": t_roof / statistics.median(cold)}
        if std and c.layers > 1 and c.B * c.N < 100000:
            # L layers, each with its own input and output buffers, in one graph.
            layers = [buffers(c, c.qkv(i % c.calls)) for i in range(c.layers)]
            side = torch.cuda.Stream(dev)
            side.wait_stream(torch.cuda.current_stream(dev))
            with torch.cuda.stream(side):
                for q_, o_ in layers:
                    call(c, q_, o_)
            torch.cuda.current_stream(dev).wait_stream(side)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=side):
                for q_, o_ in layers:
                    call(c, q_, o_)
            for _ in range(5):
                graph.replay()
            torch.cuda.synchronize()
            reps = []
            for _ in range(50):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                graph.replay()
                e1.record()
                e1.synchronize()
                reps.append(e0.elapsed_time(e1) * 1e3)
            t = statistics.median(reps)
            rec["graph_layers"] = c.layers
            rec["graph_us"] = {"median": t, "p95": _percentile(reps, 0.95),
                               "per_layer": t / c.layers}
            rec["graph_images_per_s"] = c.B / (t * 1e-6)
            rec["graph_frac"] = t_roof * c.layers / t
            del graph, layers
        print(json.dumps(rec), flush=True)
        del qkv, out
        torch.cuda.empty_cache()

    c = WORKLOAD
    bits = si.packed_qkv(1, c.N, c.H, c.d, c.seed(0))
    flops1 = 4.0 * c.H * c.N * c.N * c.d
    for threads in (oracle.default_threads(), 1):
        t0 = time.perf_counter()
        oracle.attention_packed_bf16(bits, c.scale, threads=threads)
        dt = time.perf_counter() - t0
        print(json.dumps({"mode": "configs", "oracle": "fp64 C++", "cores": threads,
                          "sample": f"1 image x {c.H} heads of {c.name}",
                          "seconds": dt, "tflops": flops1 / dt / 1e12}), flush=True)


def _graph_time_us(fn, reps: int = 20, iters: int = 10) -> list[float]:
    """Per-call times (us) of ``fn`` captured ``reps`` times back to back in one CUDA
    graph, over ``iters`` replays (the host cost of a call does not idle the GPU)."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for _ in range(reps):
            fn()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    out = []
    for _ in range(iters):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        e1.synchronize()
        out.append(e0.elapsed_time(e1) * 1e3 / reps)
    del g
    return out


def run_block(args) -> None:
    """The layers around the attention core on the encoder shapes and the bench batch:
    LayerNorm, the fused residual add + LayerNorm, the qkv linear, the output projection
    with the residual add, the MLP's fc1 + GELU and fc2 + residual; the attention half of
    a ViT block and the whole pre-norm encoder layer (LN1 -> qkv -> attention -> output
    projection + residual -> LN2 -> fc1 + GELU -> fc2 + residual), one layer at the bench
    batch, and for the encoder workloads their L layers (fresh weights and activations per
    layer) in one CUDA graph."""
    import math as _m

    import torch

    import vit_self_attention_b200 as vab

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = measured_peaks()
    p_bf16 = float(peaks["bf16_tflops"]) * 1e12
    hbm = float(peaks["hbm_gbs"]) * 1e9
    ws = torch.empty(vab.vla_linear_workspace_bytes(), dtype=torch.uint8, device=dev)
    mlp_width = {768: 3072, 1024: 4096, 1152: 4304}

    def t_(shape, mean=0.0, std=1.0, seed=1):
        b = si.normal_bf16(seed, shape, mean, std)
        return torch.from_numpy(b.view(np.int16)).to(dev).view(torch.bfloat16)

    def layer_weights(W, F, seed):
        return {"g": t_((W,), 1.0, 0.1, seed), "be": t_((W,), 0.0, 0.1, seed + 1),
                "wq": t_((3 * W, W), 0.0, 1.0 / _m.sqrt(W), seed + 2),
                "bq": t_((3 * W,), 0.0, 0.1, seed + 3),
                "wo": t_((W, W), 0.0, 1.0 / _m.sqrt(W), seed + 4), "bo": t_((W,), 0.0, 0.1, seed + 5),
                "g2": t_((W,), 1.0, 0.1, seed + 6), "be2": t_((W,), 0.0, 0.1, seed + 7),
                "w1": t_((F, W), 0.0, 1.0 / _m.sqrt(W), seed + 8), "b1": t_((F,), 0.0, 0.1, seed + 9),
                "w2": t_((W, F), 0.0, 1.0 / _m.sqrt(F), seed + 10), "b2": t_((W,), 0.0, 0.1, seed + 11)}

    for c in list(si.ENCODER_WORKLOADS[1:]) + [si.VIT_L14_336PX_B256]:
        W = c.H * c.d
        F = mlp_width[W]
        M = c.B * c.N
        x = t_((c.B, c.N, W), 0.0, 1.0, 11)
        p = layer_weights(W, F, 12)
        xn = torch.empty_like(x)
        qkv = torch.empty((c.B, c.N, 3 * W), dtype=torch.bfloat16, device=dev)
        o = torch.empty((c.B, c.N, c.H, c.d), dtype=torch.bfloat16, device=dev)
        y = torch.empty_like(x)
        s2 = torch.empty_like(x)
        a = torch.empty((c.B, c.N, F), dtype=torch.bfloat16, device=dev)
        y2 = torch.empty_like(x)
        ln = lambda: vab.layernorm(x, p["g"], p["be"], 1e-6, out=xn)
        lq = lambda: vab.linear(xn, p["wq"], p["bq"], out=qkv, workspace=ws)
        at = lambda: vab.attention(qkv.view(c.B, c.N, 3, c.H, c.d), c.scale, out=o)
        lo = lambda: vab.linear(o.view(c.B, c.N, W), p["wo"], p["bo"], x, out=y, workspace=ws)
        ln2 = lambda: vab.layernorm(y, p["g2"], p["be2"], 1e-6, out=xn)
        f1 = lambda: vab.linear_gelu(xn, p["w1"], p["b1"], out=a, workspace=ws)
        f2 = lambda: vab.linear(a, p["w2"], p["b2"], y, out=y2, workspace=ws)
        aln = lambda: vab.add_layernorm(x, y, p["g2"], p["be2"], 1e-6, out_s=s2, out_y=xn)
        ref = lambda: torch.addmm(p["bq"], xn.view(M, W), p["wq"].t(), out=qkv.view(M, 3 * W))
        big = c.B * c.N >= 100000
        reps, iters = (3, 5) if big else (20, 10)
        med = lambda f: statistics.median(_graph_time_us(f, reps, iters))
        t_ln, t_q, t_at, t_o, t_ref = med(ln), med(lq), med(at), med(lo), med(ref)
        t_f1, t_f2, t_aln = med(f1), med(f2), med(aln)
        fq, fo, ff = 2.0 * M * W * 3 * W, 2.0 * M * W * W, 2.0 * M * W * F
        rec = {"mode": "block", "workload": c.name, "tokens": M, "width": W, "mlp_width": F,
               "layernorm": {"us": t_ln, "gbs": 4.0 * M * W / t_ln / 1e3,
                             "frac_hbm": 4.0 * M * W / t_ln / 1e-6 / hbm},
               "add_layernorm": {"us": t_aln, "gbs": 8.0 * M * W / t_aln / 1e3,
                                 "frac_hbm": 8.0 * M * W / t_aln / 1e-6 / hbm},
               "qkv_linear": {"us": t_q, "tflops": fq / t_q / 1e6,
                              "frac_bf16": fq / t_q / 1e-6 / p_bf16,
                              "torch_addmm_us": t_ref},
               "attention": {"us": t_at, "tflops": c.flops() / t_at / 1e6},
               "out_linear_residual": {"us": t_o, "tflops": fo / t_o / 1e6,
                                       "frac_bf16": fo / t_o / 1e-6 / p_bf16},
               "fc1_gelu": {"us": t_f1, "tflops": ff / t_f1 / 1e6,
                            "frac_bf16": ff / t_f1 / 1e-6 / p_bf16},
               "fc2_residual": {"us": t_f2, "tflops": ff / t_f2 / 1e6,
                                "frac_bf16": ff / t_f2 / 1e-6 / p_bf16}}
        t_half = med(lambda: (ln(), lq(), at(), lo()))
        rec["half_block_us"] = t_half
        rec["half_block_tflops"] = (fq + fo + c.flops()) / t_half / 1e6
        layer_flops = fq + fo + 2.0 * ff + c.flops()
        # Seconds of back-to-back GEMMs can run into the power cap: the layer's
        # timing carries the SM clocks and throttle reasons seen while it ran.
        with ClockSampler(torch.cuda.current_device()) as clocks:
            clocks.mark_start()
            t_layer = med(lambda: (ln(), lq(), at(), lo(), ln2(), f1(), f2()))
            clocks.mark_end()
        rec["layer_us"] = t_layer
        rec["layer_clocks"] = clocks.summary()
        rec["layer_tflops"] = layer_flops / t_layer / 1e6
        if not big:
            # The encoder's L whole layers (fresh weights and activations per layer) in one
            # graph; the residual stream moves to a new buffer at every residual add.
            layers = [layer_weights(W, F, 100 + 13 * i) for i in range(c.layers)]
            xs = [x.clone() for _ in range(2 * c.layers + 1)]

            def encoder():
                for i, q in enumerate(layers):
                    h_in, h_mid, h_out = xs[2 * i], xs[2 * i + 1], xs[2 * i + 2]
                    vab.layernorm(h_in, q["g"], q["be"], 1e-6, out=xn)
                    vab.linear(xn, q["wq"], q["bq"], out=qkv, workspace=ws)
                    vab.attention(qkv.view(c.B, c.N, 3, c.H, c.d), c.scale, out=o)
                    vab.linear(o.view(c.B, c.N, W), q["wo"], q["bo"], h_in, out=h_mid,
                               workspace=ws)
                    vab.layernorm(h_mid, q["g2"], q["be2"], 1e-6, out=xn)
                    vab.linear_gelu(xn, q["w1"], q["b1"], out=a, workspace=ws)
                    vab.linear(a, q["w2"], q["b2"], h_mid, out=h_out, workspace=ws)

            t_enc = statistics.median(_graph_time_us(encoder, 1, 20))
            rec["encoder_layers"] = c.layers
            rec["encoder_us"] = t_enc
            rec["encoder_tflops"] = c.layers * layer_flops / t_enc / 1e6
            rec["encoder_images_per_s"] = c.B / (t_enc * 1e-6)
            del layers, xs
        print(json.dumps(rec), flush=True)
        del x, xn, qkv, o, y, s2, a, y2, p
        torch.cuda.empty_cache()


def run_layer(args) -> None:
    """One whole pre-norm encoder layer of a named workload (LN1 -> qkv -> attention ->
    output projection + residual -> LN2 -> fc1 + GELU -> fc2 + residual), seeded weights
    and activations, launched eagerly stage by stage: three warm layers, then ten timed
    ones with CUDA events around every stage (one JSON line of per-stage medians).  Its
    launches in stream order are what an ncu launch list of one layer shows."""
    import math as _m

    import torch

    import vit_self_attention_b200 as vab

    names = {c.name: c for c in list(si.ENCODER_WORKLOADS) + [si.VIT_L14_336PX_B256]}
    if args.layer not in names:
        raise SystemExit(f"--layer: one of {sorted(names)}")
    c = names[args.layer]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    W = c.H * c.d
    F = {768: 3072, 1024: 4096, 1152: 4304}[W]

    def t_(shape, mean=0.0, std=1.0, seed=1):
        b = si.normal_bf16(seed, shape, mean, std)
        return torch.from_numpy(b.view(np.int16)).to(dev).view(torch.bfloat16)

    g, be = t_((W,), 1.0, 0.1, 12), t_((W,), 0.0, 0.1, 13)
    wq, bq = t_((3 * W, W), 0.0, 1.0 / _m.sqrt(W), 14), t_((3 * W,), 0.0, 0.1, 15)
    wo, bo = t_((W, W), 0.0, 1.0 / _m.sqrt(W), 16), t_((W,), 0.0, 0.1, 17)
    g2, be2 = t_((W,), 1.0, 0.1, 18), t_((W,), 0.0, 0.1, 19)
    w1, b1 = t_((F, W), 0.0, 1.0 / _m.sqrt(W), 20), t_((F,), 0.0, 0.1, 21)
    w2, b2 = t_((W, F), 0.0, 1.0 / _m.sqrt(F), 22), t_((W,), 0.0, 0.1, 23)
    x = t_((c.B, c.N, W), 0.0, 1.0, 11)
    xn = torch.empty_like(x)
    qkv = torch.empty((c.B, c.N, 3 * W), dtype=torch.bfloat16, device=dev)
    o = torch.empty((c.B, c.N, c.H, c.d), dtype=torch.bfloat16, device=dev)
    y = torch.empty_like(x)
    a = torch.empty((c.B, c.N, F), dtype=torch.bfloat16, device=dev)
    y2 = torch.empty_like(x)
    ws = torch.empty(vab.vla_linear_workspace_bytes(), dtype=torch.uint8, device=dev)
    stages = [
        ("layernorm_1", lambda: vab.layernorm(x, g, be, 1e-6, out=xn)),
        ("qkv_linear", lambda: vab.linear(xn, wq, bq, out=qkv, workspace=ws)),
        ("attention", lambda: vab.attention(qkv.view(c.B, c.N, 3, c.H, c.d), c.scale, out=o)),
        ("out_linear_residual",
         lambda: vab.linear(o.view(c.B, c.N, W), wo, bo, x, out=y, workspace=ws)),
        ("layernorm_2", lambda: vab.layernorm(y, g2, be2, 1e-6, out=xn)),
        ("fc1_gelu", lambda: vab.linear_gelu(xn, w1, b1, out=a, workspace=ws)),
        ("fc2_residual", lambda: vab.linear(a, w2, b2, y, out=y2, workspace=ws)),
    ]
    for _ in range(3):
        for _, f in stages:
            f()
    torch.cuda.synchronize()
    times = {n: [] for n, _ in stages}
    for _ in range(10):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)]
        evs[0].record()
        for i, (_, f) in enumerate(stages):
            f()
            evs[i + 1].record()
        evs[-1].synchronize()
        for i, (n, _) in enumerate(stages):
            times[n].append(evs[i].elapsed_time(evs[i + 1]) * 1e3)
    med = {n: statistics.median(v) for n, v in times.items()}
    total = sum(med.values())
    print(json.dumps({"mode": "layer", "workload": c.name, "tokens": c.B * c.N,
                      "stage_us": med, "layer_us": total,
                      "share": {n: v / total for n, v in med.items()}}), flush=True)


def run_linear(args) -> None:
    """One linear layer y = x w^T + bias (+ a residual, or GELU) on an (M, K, N) shape with
    seeded bf16 operands: five warm calls, then the median of 20 CUDA-event timed calls
    (one JSON line).  Small enough to run under ncu (the GEMM's profile)."""
    import math as _m

    import torch

    import vit_self_attention_b200 as vab

    fields = args.linear.split(",")
    M, K, N = (int(v) for v in fields[:3])
    epi = fields[3] if len(fields) > 3 else "bias"
    if epi not in ("bias", "res", "gelu"):
        raise SystemExit("--linear M,K,N[,bias|res|gelu]")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)

    def t_(shape, std, seed):
        b = si.normal_bf16(seed, shape, 0.0, std)
        return torch.from_numpy(b.view(np.int16)).to(dev).view(torch.bfloat16)

    x, w, b = t_((M, K), 1.0, 21), t_((N, K), 1.0 / _m.sqrt(K), 22), t_((N,), 0.1, 23)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    r = t_((M, N), 1.0, 24) if epi == "res" else None
    ws = torch.empty(vab.vla_linear_workspace_bytes(), dtype=torch.uint8, device=dev)

    def call():
        if epi == "gelu":
            vab.linear_gelu(x, w, b, out=y, workspace=ws)
        else:
            vab.linear(x, w, b, res=r, out=y, workspace=ws)

    for _ in range(5):
        call()
    torch.cuda.synchronize()
    ts = []
    for _ in range(20):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        e1.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
    us = statistics.median(ts)
    peaks = measured_peaks()
    print(json.dumps({"mode": "linear", "M": M, "K": K, "N": N, "epilogue": epi, "us": us,
                      "tflops": 2.0 * M * N * K / us / 1e6,
                      "frac_bf16": 2.0 * M * N * K / us / 1e-6 / (peaks["bf16_tflops"] * 1e12),
                      "peak_source": peaks["source"]}), flush=True)


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target duration of the CPU oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--images", type=int, default=None,
                    help="override B (profiling captures of a smaller case of the same kernel)")
    ap.add_argument("--configs", action="store_true",
                    help="per-config report instead of the benchmark line (1 GPU)")
    ap.add_argument("--block", action="store_true",
                    help="the layers around attention, whole encoder layers and encoders (1 GPU)")
    ap.add_argument("--layer", default=None, metavar="WORKLOAD",
                    help="one whole encoder layer of a workload, stage by stage (1 GPU)")
    ap.add_argument("--linear", default=None, metavar="M,K,N[,bias|res|gelu]",
                    help="time one linear layer y = x w^T + bias (+ residual, or GELU) of this "
                         "shape (1 GPU)")
    args = ap.parse_args()
    if args.configs:
        run_configs(args)
        return
    if args.block:
        run_block(args)
        return
    if args.linear:
        run_linear(args)
        return
    if args.layer:
        run_layer(args)
        return

    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        if args.impl == "reference":
            # The CPU oracle runs on rank 0 alone; the other ranks would do no work.
            run_reference(args, 0, args.gpus)
            return
        # No outer torchrun: start one process per GPU here (same per-rank batch, NCCL
        # process group over 127.0.0.1), so that --gpus N alone measures N GPUs.
        launch_ranks(args.gpus, _rank_main, args, backend="nccl")
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and world > 1:
        print(f"warning: WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    if world > 1:
        init_group("nccl", rank, world, local_rank)
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


def init_group(backend: str, rank: int, world: int, local_rank: int) -> None:
    """Join the job's process group (MASTER_ADDR / MASTER_PORT from the environment) with
    a short timeout, so that ranks waiting on a lost peer end with an error."""
    import datetime

    import torch
    import torch.distributed as dist
    timeout = datetime.timedelta(seconds=120)
    if backend == "nccl":
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", rank=rank, world_size=world, timeout=timeout,
                                device_id=torch.device("cuda", local_rank))
    else:
        dist.init_process_group(backend, rank=rank, world_size=world, timeout=timeout)


def _free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank_entry(rank: int, world: int, port: int, backend: str, target, target_args) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    init_group(backend, rank, world, rank)
    try:
        target(rank, world, *target_args)
    finally:
        dist.destroy_process_group()


def launch_ranks(nprocs: int, target, *target_args, backend: str = "nccl") -> None:
    """Run ``target(rank, world, *target_args)`` in ``nprocs`` spawned processes that form
    one process group (rank r on GPU r for NCCL); raises if any rank fails."""
    import torch.multiprocessing as mp
    mp.spawn(_rank_entry, args=(nprocs, _free_port(), backend, target, target_args),
             nprocs=nprocs, join=True)


def _rank_main(rank: int, world: int, args) -> None:
    run_ours(args, rank, world, rank)


if __name__ == "__main__":
    main()

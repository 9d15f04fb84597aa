#!/usr/bin/env python3
"""Throughput of the KroQuant online activation quantizer on B200.

One step = one pass of the whole hot path (load, block transform, amax, E8M0
scale, E2M1 round, pack, store) over the FLUX.1-schnell-shaped activations of
one denoising step: M = 4608 tokens at d = 3072 and at d = 12288 (bf16, Student-t
nu = 3, 0.5 % outlier channels x100, seeded synthetic data).  The metric is
quantizer GB/s with algorithmic bytes (2 B in + 0.5 B codes + 1/32 B scales per
element), its fraction of HBM bandwidth, and tokens/s.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
  python bench.py --sweep   # KroQuant vs per-channel scaling vs FWHT, every shape

Multi-GPU (torchrun, one process per GPU): rows are independent, each rank
quantizes its own batch (weak scaling, no collective on the data path); time is
the max over ranks.  ``--impl reference`` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mxfp4_activations_b200 import inputs  # noqa: E402

FLUX_M = 4608
FLUX_DS = (3072, 12288)
BYTES_PER_ELEM = 2.0 + 0.5 + 1.0 / 32.0
PROFILE_JSON = os.path.join(ROOT, "profiles", "kq_quant_flux_traffic.json")
FLUX_WORKLOAD = ("FLUX.1-schnell-shaped activations, M=4608 tokens x d in {3072, 12288} bf16, "
                 "Student-t(3) with 0.5% outlier channels x100, per-block LU params Hadamard+N(0,0.05)")

KERNEL_SOURCES = ["mxfp4_activations_b200/csrc/kq_quant.cuh", "mxfp4_activations_b200/csrc/kq_common.cuh",
                  "mxfp4_activations_b200/csrc/kq_mx.cuh"]


def algo_bytes(M: int, d: int) -> float:
    return BYTES_PER_ELEM * M * d


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


FP4_OVER_BF16 = 4.0  # nominal dense ratio on B200: 9 PFLOP/s FP4 / 2.25 PFLOP/s bf16


def gemm_leg(torch, kq, n: int, device) -> dict:
    """The quantizer's consumer, kq_gemm_mxf4 (bf16 C), on the FLUX linear-layer
    shapes: random MXFP4 operands, four copies of each rotated so that the operands
    of consecutive launches are not all in L2, back-to-back launches between CUDA
    events.  cuBLAS's block-scaled FP4 GEMM (through torch) on the same operands
    is timed beside it as a cross-check."""
    F = torch.nn.functional
    peaks = measured_peaks()
    peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    out = {"peak_tflops": round(peak, 1),
           "peak_source": f"{peaks['source']} bf16 burst x {FP4_OVER_BF16:g} (nominal FP4/bf16 ratio)",
           "output": "bf16", "timing": f"{n} launches back to back over 4 rotated operand copies", "shapes": {}}
    for name, (M, N, K) in inputs.GEMM_SHAPES.items():
        sets = []
        for c in range(4):
            aq, _ = inputs.mx_operand(M, K, seed=[M, N, K, c, 1])
            bq, _ = inputs.mx_operand(N, K, seed=[M, N, K, c, 2])
            rng = np.random.default_rng([M, N, K, c, 3])
            sa = rng.integers(118, 137, kq.scale_bytes(M, K, "mma"), dtype=np.uint8)
            sb = rng.integers(118, 137, kq.scale_bytes(N, K, "mma"), dtype=np.uint8)
            sets.append([torch.from_numpy(a).to(device) for a in (aq, sa, bq, sb)])
        C = torch.empty((M, N), dtype=torch.bfloat16, device=device)

        def ours(i):
            a, sa_, b, sb_ = sets[i % 4]
            kq.kq_gemm_mxf4(a, sa_, b, sb_, out=C)

        def cublas(i):
            a, sa_, b, sb_ = sets[i % 4]
            F.scaled_mm(a.view(torch.float4_e2m1fn_x2), b.view(torch.float4_e2m1fn_x2).t(),
                        sa_.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                        sb_.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                        swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                        output_dtype=torch.bfloat16)

        def loop(fn) -> float:
            for i in range(8):
                fn(i)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for i in range(n):
                fn(i)
            e1.record()
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) * 1e3 / n

        flops = 2.0 * M * N * K
        us = loop(ours)
        rec = {"M": M, "N": N, "K": K, "us": round(us, 2), "tflops": round(flops / us / 1e6, 1),
               "frac": round(flops / us / 1e6 / peak, 4)}
        try:
            cus = loop(cublas)
            rec["cublas_us"] = round(cus, 2)
            rec["cublas_tflops"] = round(flops / cus / 1e6, 1)
        except (RuntimeError, AttributeError, TypeError, ValueError) as e:
            rec["cublas_us"] = f"unavailable: {str(e).splitlines()[0][:80]}"
        out["shapes"][name] = rec
        del sets, C
    err = kq.kq_get_device_error(clear=True)
    if err != 0:
        raise RuntimeError(f"device error in the GEMM leg: {kq.kq_status_string(err)}")
    return out


def recorded_exact_path_share():
    """Share of blocks the certified kernels send to their exact path at the bench's
    FLUX inputs: the host estimate committed by tests/exact_path_rate.py."""
    path = os.path.join(ROOT, "profiles", "kq_exact_path_rate.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    return {"kind": "host estimate (tests/exact_path_rate.py)",
            "butterfly": {d: round(r["butterfly"], 5) for d, r in rec["rates"].items()},
            "tensor_core_bf16_K": {d: round(r["tensor_core_bf16_K"], 5) for d, r in rec["rates"].items()},
            "tensor_core_fp32_K": {d: round(r["tensor_core_fp32_K"], 5) for d, r in rec["rates"].items()}}


def recorded_traffic(d: int):
    """DRAM bytes (read + write) of one launch of the dominant kernel at width d,
    from the committed ncu summary, if it was taken on the current kernel sources;
    else None."""
    if not os.path.exists(PROFILE_JSON):
        return None
    with open(PROFILE_JSON) as f:
        rec = json.load(f)
    if rec.get("source_hash") != kernel_source_hash():
        return None
    for launch in rec.get("launches", []):
        if launch.get("d") == d:
            return launch["dram_read_bytes"] + launch["dram_write_bytes"]
    return None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self) -> dict:
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[3:7]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- ranks

def rank_inputs(rank: int):
    """The FLUX-shaped batch of one rank: rank 0 uses the configuration's own
    seed, every other rank draws an independent batch of the same shape and law
    (weak scaling: work per rank is fixed).  The transform parameters are the
    layer's and are the same on every rank."""
    xs, ps = [], []
    for d in FLUX_DS:
        x, p = inputs.config_case("flux", d)
        if rank:
            x = inputs.activations(FLUX_M, d, "t3", seed=[3, d, 0, rank], outlier_frac=0.005,
                                   outlier_scale=(100.0, 100.0))
        xs.append(x)
        ps.append(p)
    return xs, ps


def max_over_ranks(ms: float, dist, device) -> float:
    """Elapsed time of the job: the slowest rank's time (one scalar all-reduce)."""
    import torch

    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- GPU arm

class QuantStep:
    """Device-resident buffers for one step over every d, rotated over n copies."""

    def __init__(self, torch, kq, xs_host, params_host, n_copies: int, device):
        self.torch = torch
        self.kq = kq
        self.lib = kq.load()
        self.items = []
        for d, x, params in zip(FLUX_DS, xs_host, params_host):
            p = torch.from_numpy(params).to(device)
            mats = kq.kq_expand_blocks(p)
            mats16 = kq.kq_expand_blocks(p, dtype=torch.bfloat16)
            fac = kq.kq_expand_factored(p)
            x0 = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
            copies = [x0] + [x0.clone() for _ in range(n_copies - 1)]
            M = x.shape[0]
            qs = [torch.empty((M, d // 2), dtype=torch.uint8, device=device) for _ in range(n_copies)]
            ss = [torch.empty((M, d // 32), dtype=torch.uint8, device=device) for _ in range(n_copies)]
            inv_s = torch.from_numpy(inputs.smooth_inv_scale(x)).to(device)
            # AdaLN modulation vectors of two samples of M/2 tokens (the fused producer's input)
            rng = np.random.default_rng([d, 77])
            mod = [torch.from_numpy(inputs.f32_to_bf16_bits((sd * rng.standard_normal((2, d))).astype(np.float32))
                                    .view(np.int16)).to(device) for sd in (0.5, 0.3)]
            stats = torch.empty((M, 2), dtype=torch.float32, device=device)
            self.items.append(dict(d=d, M=M, params=p, mats=mats, mats16=mats16, fac=fac, x=copies, q=qs, s=ss,
                                   inv_s=inv_s, shift=mod[0], scale=mod[1], stats=stats))
        self.n = n_copies
        self.stream = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)

    def launch(self, it: int, item: dict, kind: str = "kroquant"):
        c = it % self.n
        x, q, s = item["x"][c], item["q"][c], item["s"][c]
        M, d = item["M"], item["d"]
        if kind == "kroquant":
            st = self.lib.kq_quantize(x.data_ptr(), M, d, d, item["mats"].data_ptr(), 0, item["fac"].data_ptr(),
                                      q.data_ptr(), s.data_ptr(), 2, 0, self.stream)
        elif kind == "kroquant_mma":
            st = self.lib.kq_quantize(x.data_ptr(), M, d, d, item["mats"].data_ptr(), 0, None,
                                      q.data_ptr(), s.data_ptr(), 1, 0, self.stream)
        elif kind == "kroquant_mma_bf16":
            st = self.lib.kq_quantize(x.data_ptr(), M, d, d, item["mats16"].data_ptr(), 1, None,
                                      q.data_ptr(), s.data_ptr(), 1, 0, self.stream)
        elif kind in ("kroquant_adaln", "kroquant_adaln_fused"):
            # with a statistics buffer: the statistics pass, then the quantizer's AdaLN form;
            # without one: the single fused kernel
            stats = item["stats"].data_ptr() if kind == "kroquant_adaln" else None
            st = self.lib.kq_adaln_quantize(x.data_ptr(), M, d, d, item["shift"].data_ptr(), item["scale"].data_ptr(),
                                            (M + 1) // 2, ctypes.c_float(1e-6), item["mats"].data_ptr(),
                                            item["fac"].data_ptr(), q.data_ptr(), s.data_ptr(), 0, stats, self.stream)
        elif kind == "smooth":
            st = self.lib.kq_ref_smooth_quantize(x.data_ptr(), M, d, d, item["inv_s"].data_ptr(), q.data_ptr(),
                                                 s.data_ptr(), self.stream)
        else:
            st = self.lib.kq_ref_fwht_quantize(x.data_ptr(), M, d, d, q.data_ptr(), s.data_ptr(), self.stream)
        if st != 0:
            raise RuntimeError(f"{kind} launch failed: {self.lib.kq_status_string(st).decode()}")

    def bytes_per_step(self) -> float:
        return sum(algo_bytes(it["M"], it["d"]) for it in self.items)


def timed(torch, step: QuantStep, K: int, kind: str, per_launch: bool):
    """K steps bracketed by events; optional events around every launch."""
    ev = torch.cuda.Event
    if per_launch:
        marks = [[(ev(enable_timing=True), ev(enable_timing=True)) for _ in step.items] for _ in range(K)]
    start, stop = ev(enable_timing=True), ev(enable_timing=True)
    start.record()
    for it in range(K):
        for j, item in enumerate(step.items):
            if per_launch:
                marks[it][j][0].record()
            step.launch(it, item, kind)
            if per_launch:
                marks[it][j][1].record()
    stop.record()
    stop.synchronize()
    total_ms = start.elapsed_time(stop)
    launch_ms = None
    if per_launch:
        launch_ms = [sum(a.elapsed_time(b) for a, b in (marks[i][j] for i in range(K))) for j in range(len(step.items))]
    return total_ms, launch_ms


def timed_b2b(torch, step: QuantStep, j: int, kind: str, K: int) -> float:
    """Average duration (microseconds) of one launch of `kind` on item j (one d),
    from K launches queued back to back on the launching stream with CUDA events
    around the whole loop (inputs rotate over the resident copies, so every launch
    reads from HBM)."""
    item = step.items[j]
    for it in range(3):
        step.launch(it, item, kind)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for it in range(K):
        step.launch(it, item, kind)
    b.record()
    b.synchronize()
    return a.elapsed_time(b) * 1e3 / K


def e2e_run(torch, kq, step: QuantStep, xs_host, K: int):
    """Same metric through the public API with host buffers: every step copies
    that step's activations from pinned host memory, quantizes them, and reads the
    codes and scales back to pinned host memory.  The three run on their own
    streams (upload, compute, download) with double-buffered device and host
    buffers, so step i's upload overlaps step i-1's quantizer and download."""
    dev = step.items[0]["x"][0].device
    hx = [torch.from_numpy(x.view(np.int16)).pin_memory() for x in xs_host]
    hq = [[torch.empty((it["M"], it["d"] // 2), dtype=torch.uint8).pin_memory() for it in step.items]
          for _ in range(2)]
    hs = [[torch.empty((it["M"], it["d"] // 32), dtype=torch.uint8).pin_memory() for it in step.items]
          for _ in range(2)]
    dx = [[torch.empty(x.shape, dtype=torch.int16, device=dev) for x in xs_host] for _ in range(2)]
    dq = [[torch.empty((it["M"], it["d"] // 2), dtype=torch.uint8, device=dev) for it in step.items]
          for _ in range(2)]
    ds = [[torch.empty((it["M"], it["d"] // 32), dtype=torch.uint8, device=dev) for it in step.items]
          for _ in range(2)]
    h2d = sum(x.nbytes for x in xs_host)
    d2h = sum(t.numel() for t in hq[0]) + sum(t.numel() for t in hs[0])
    s_in, s_cp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev = {k: [[torch.cuda.Event() for _ in step.items] for _ in range(2)] for k in ("in", "cp", "out")}

    def issue(i: int):
        p = i % 2
        for j, it in enumerate(step.items):
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev["cp"][p][j])  # step i-2's quantizer has read dx[p][j]
                dx[p][j].copy_(hx[j], non_blocking=True)
                ev["in"][p][j].record(s_in)
            with torch.cuda.stream(s_cp):
                s_cp.wait_event(ev["in"][p][j])
                if i >= 2:
                    s_cp.wait_event(ev["out"][p][j])  # step i-2's download has read dq/ds[p][j]
                kq.kq_quantize(dx[p][j].view(torch.bfloat16), it["mats"], it["fac"], variant="butterfly",
                               q=dq[p][j], scales=ds[p][j])
                ev["cp"][p][j].record(s_cp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["cp"][p][j])
                hq[p][j].copy_(dq[p][j], non_blocking=True)
                hs[p][j].copy_(ds[p][j], non_blocking=True)
                ev["out"][p][j].record(s_out)

    def run(n: int) -> float:
        main = torch.cuda.current_stream(dev)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(main)
        for s in (s_in, s_cp, s_out):
            s.wait_stream(main)
        for i in range(n):
            issue(i)
        for s in (s_in, s_cp, s_out):
            main.wait_stream(s)
        t1.record(main)
        t1.synchronize()
        return t0.elapsed_time(t1)

    run(2)
    ms = run(K)
    return ms, h2d, d2h


def run_gpu(args) -> None:
    import torch
    import torch.distributed as dist

    import mxfp4_activations_b200 as kq
    from mxfp4_activations_b200 import build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", init_method="env://", timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local if world > 1 else 0)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    kq.load()

    xs, ps = rank_inputs(rank)
    step = QuantStep(torch, kq, xs, ps, n_copies=4, device=device)
    bytes_step = step.bytes_per_step()
    resident_mb = 4 * sum(x.nbytes for x in xs) / 1e6

    for it in range(args.warmup):
        for item in step.items:
            step.launch(it, item)
    torch.cuda.synchronize()
    err = kq.kq_get_device_error(clear=True)
    if err != 0:
        raise RuntimeError(f"device error after warm-up: {kq.kq_status_string(err)}")

    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0] or 0) if world == 1 else local
    with ClockSampler(gpu_index) as clk:
        # untimed soak so that the clock record covers a loaded GPU, then the timed K steps
        t_end = time.time() + 1.0
        it = 0
        while time.time() < t_end:
            for item in step.items:
                step.launch(it, item)
            it += 1
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        # the K timed steps, back to back: events only around the whole loop (events
        # between launches would serialise them and cost ~14 us per step)
        total_ms, _ = timed(torch, step, args.steps, "kroquant", per_launch=False)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        # the dominant kernel (the d = 12288 launch) alone, back to back: its average
        # launch duration for the roofline
        dom = max(range(len(step.items)), key=lambda j: step.items[j]["d"])
        dom_us = timed_b2b(torch, step, dom, "kroquant", args.steps)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        # the K steps once more with events around every launch (these serialise the
        # launches and add each launch's start-up; reported beside the roofline)
        _, launch_ms = timed(torch, step, args.steps, "kroquant", per_launch=True)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    if world > 1:
        total_ms = max_over_ranks(total_ms, dist, device)

    err = kq.kq_get_device_error(clear=True)
    if err != 0:
        raise RuntimeError(f"device error in timed region: {kq.kq_status_string(err)}")

    # comparison kernels on the same inputs (after the timed region): every kind,
    # each shape back to back on its own
    comp = {}
    n_cmp = max(50, args.steps)
    for kind in ("smooth", "fwht", "kroquant", "kroquant_mma", "kroquant_mma_bf16", "kroquant_adaln",
                 "kroquant_adaln_fused"):
        us = {str(it["d"]): timed_b2b(torch, step, j, kind, n_cmp) for j, it in enumerate(step.items)}
        comp[kind] = {"gbs": bytes_step / (sum(us.values()) * 1e-6) / 1e9, "us_per_launch": us}

    gemm = gemm_leg(torch, kq, max(20, min(args.steps, 50)), device)

    e2e_steps = max(3, min(args.steps, 20))
    e2e_ms, h2d, d2h = e2e_run(torch, kq, step, xs, e2e_steps)
    if world > 1:
        e2e_ms = max_over_ranks(e2e_ms, dist, device)

    if world > 1:
        dist.barrier()
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    peaks = measured_peaks()
    value = world * bytes_step * args.steps / (total_ms * 1e-3) / 1e9
    dom_item = step.items[dom]
    dom_bytes = algo_bytes(dom_item["M"], dom_item["d"])
    achieved = dom_bytes / (dom_us * 1e-6) / 1e9
    traffic = recorded_traffic(dom_item["d"])
    clocks = clk.summary()
    out = {
        "metric": "quantizer GB/s (bf16 in + FP4/E8M0 out) and % of B200 HBM peak; tokens/s",
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {
            "workload": FLUX_WORKLOAD,
            "M": FLUX_M, "d": list(FLUX_DS), "variant": "butterfly",
            "l2": f"inputs rotated over 4 device copies ({resident_mb:.0f} MB > 126 MB L2)",
            "parallelism": f"dp{world} (rows sharded, no collective)",
        },
        "tokens_per_s": round(world * FLUX_M * args.steps / (total_ms * 1e-3), 1),
        "hbm_frac_measured": round(value / world / peaks["hbm_gbs"], 4),
        "hbm_frac_nominal_8tbs": round(value / world / 8000.0, 4),
        "roofline": {
            "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4), "peak_source": peaks["source"],
            "traffic": traffic,
            "kernel": "quant_kernel<MODE_KRON, row-major scales, 32-element blocks>",
            "launch": f"M={dom_item['M']}, d={dom_item['d']}",
            "algorithmic_bytes_per_launch": dom_bytes,
            "us_per_launch": round(dom_us, 3),
            "timing": f"{args.steps} launches of this kernel back to back, CUDA events around the loop",
            "us_per_launch_serialised": {str(it["d"]): round(launch_ms[j] * 1e3 / args.steps, 3)
                                         for j, it in enumerate(step.items)},
        },
        "comparison": {k: {"gbs": round(v["gbs"], 1),
                           "us_per_launch": {dk: round(dv, 3) for dk, dv in v["us_per_launch"].items()}}
                       for k, v in comp.items()},
        "e2e": {"value": round(world * bytes_step * e2e_steps / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "tokens_per_s": round(world * FLUX_M * e2e_steps / (e2e_ms * 1e-3), 1),
                "streams": "upload / quantize / download overlapped across steps, double-buffered"},
        "gpu_launches": len(FLUX_DS) * args.steps,
        "clocks": clocks,
        "gemm_w4a4": gemm,
        "exact_path_share": recorded_exact_path_share(),
    }
    if not args.no_cpu_baseline and world == 1:
        out["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------- CPU oracle (baseline / reference arm)

def flux_oracle_data():
    from oracle import oracle as orc

    orc.build()
    data = []
    for d in FLUX_DS:
        x, p = inputs.config_case("flux", d)
        data.append((x, orc.expand(p)))
    return data


def oracle_sample(seconds: float, data=None):
    """Time the oracle on the leading rows of the same FLUX workload; the row
    count grows (up to all M rows, then whole repeated passes) until the sample
    takes about `seconds` of single-thread CPU work."""
    from oracle import oracle as orc

    data = data or flux_oracle_data()
    rows, passes = 8, 1
    while True:
        t0 = time.perf_counter()
        for _ in range(passes):
            for x, K in data:
                orc.quantize(np.ascontiguousarray(x[:rows]), K)
        dt = time.perf_counter() - t0
        if dt >= 0.8 * seconds:
            break
        grow = seconds / max(dt, 1e-3) * 1.05
        if rows < FLUX_M:
            rows = min(FLUX_M, max(rows * 2, int(rows * grow)))
        else:
            passes = max(passes + 1, int(passes * grow))
    nbytes = sum(algo_bytes(rows, d) for d in FLUX_DS) * passes
    return nbytes / dt / 1e9, rows, passes, dt


_POOL_DATA = None


def _pool_init():
    global _POOL_DATA
    _POOL_DATA = flux_oracle_data()


def _pool_work(task):
    """One worker's share: `passes` passes over rows [r0, r0 + rows) of each FLUX shape."""
    from oracle import oracle as orc

    r0, rows, passes = task
    for _ in range(passes):
        for x, K in _POOL_DATA:
            orc.quantize(np.ascontiguousarray(x[r0:r0 + rows]), K)
    return rows * passes


def oracle_workers() -> int:
    return max(1, min(os.cpu_count() or 1, 16))


class OraclePool:
    """The unmodified oracle in one process per host core (spawned, so it is safe
    after CUDA has been initialised); rows are split across the workers."""

    def __init__(self, workers: int):
        import multiprocessing

        self.n = workers
        self.pool = multiprocessing.get_context("spawn").Pool(workers, initializer=_pool_init)
        self.pool.map(_pool_work, [(0, 1, 1)] * workers, chunksize=1)  # every worker has its data

    def run(self, rows: int, passes: int) -> float:
        """All workers at once; returns algorithmic bytes processed."""
        rows = min(rows, FLUX_M)
        tasks = [((i * rows) % (FLUX_M - rows + 1), rows, passes) for i in range(self.n)]
        self.pool.map(_pool_work, tasks, chunksize=1)
        return sum(algo_bytes(rows, d) for d in FLUX_DS) * passes * self.n

    def close(self):
        self.pool.close()
        self.pool.join()


def cpu_baseline(seconds: float) -> dict:
    gbs1, rows, passes, dt1 = oracle_sample(seconds)
    pool = OraclePool(oracle_workers())
    try:
        t0 = time.perf_counter()
        nbytes = pool.run(rows, passes)
        dt = time.perf_counter() - t0
    finally:
        pool.close()
    return {"value": round(nbytes / dt / 1e9, 6), "unit": "GB/s", "cores": pool.n, "kind": "oracle",
            "sample": f"{pool.n} processes, each {passes} pass(es) over {rows} of 4608 rows of each FLUX shape "
                      f"(d=3072 and d=12288), {dt:.1f} s wall of the C oracle, same algorithmic-byte numerator",
            "single_thread": {"value": round(gbs1, 6), "unit": "GB/s", "seconds": round(dt1, 1)}}


def run_reference(args) -> None:
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # each step: a bounded sample of the workload, sized so that W + K steps end in minutes
    per_step = max(0.5, min(10.0, 120.0 / max(1, args.steps + args.warmup)))
    data = flux_oracle_data()
    _, rows, passes, _ = oracle_sample(per_step, data)
    pool = OraclePool(oracle_workers())
    try:
        for _ in range(args.warmup):
            pool.run(rows, passes)
        t0 = time.perf_counter()
        nbytes = 0.0
        for _ in range(args.steps):
            nbytes += pool.run(rows, passes)
        dt = time.perf_counter() - t0
    finally:
        pool.close()
    gbs = nbytes / dt / 1e9
    sample = (f"{pool.n} processes per step, each {passes} pass(es) over {rows} rows of each FLUX shape "
              f"(d=3072, d=12288), C oracle")
    out = {
        "impl": "reference",
        "metric": "quantizer GB/s (bf16 in + FP4/E8M0 out) and % of B200 HBM peak; tokens/s",
        "value": round(gbs, 6), "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3 / max(1, args.steps), 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": FLUX_WORKLOAD, "M": FLUX_M, "d": list(FLUX_DS)},
        "tokens_per_s": round(rows * passes * pool.n * args.steps / dt, 3),
        "cpu_baseline": {"value": round(gbs, 6), "unit": "GB/s", "cores": pool.n, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(gbs, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


# ---------------------------------------------------------------- sweep (config 4 and the named configs)

def graph_time(torch, fn, n: int) -> float:
    """Microseconds per launch of `n` back-to-back calls of fn(stream) captured in one CUDA graph."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        assert fn(ctypes.c_void_p(side.cuda_stream)) == 0
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        for _ in range(n):
            assert fn(st) == 0
    for _ in range(3):
        g.replay()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(10):
        g.replay()
    b.record()
    b.synchronize()
    del g
    return a.elapsed_time(b) * 1e3 / (10 * n)


def run_sweep(args) -> None:
    """Every quantizer kind on every named config and sweep shape: average launch
    duration over launches queued back to back (CUDA events around the loop).
    Inputs rotate over enough device copies that a loop touches more than 256 MB
    (so each launch reads from HBM) unless a copy is under 1 MB (launch-bound
    shapes, where the inputs stay in L2 as they would in use)."""
    import torch

    import mxfp4_activations_b200 as kq
    from mxfp4_activations_b200 import build

    build.build()
    lib = kq.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [(name, M, d) for name, c in inputs.CONFIGS.items() for d in c["ds"] for M in [c["M"]]]
    cases += [("sweep", M, d) for M in inputs.SWEEP_M for d in inputs.SWEEP_D]
    for name, M, d in cases:
        x, p = inputs.sweep_case(M, d) if name == "sweep" else inputs.config_case(name, d)
        nbytes = x.nbytes
        ncopy = 1 if nbytes < 2**20 else max(1, min(8, -(-(256 * 2**20) // nbytes)))
        x0 = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
        xs = [x0] + [x0.clone() for _ in range(ncopy - 1)]
        pd = torch.from_numpy(p).cuda()
        mats, fac = kq.kq_expand_blocks(pd), kq.kq_expand_factored(pd)
        inv_s = torch.from_numpy(inputs.smooth_inv_scale(x)).cuda()
        q = torch.empty((M, d // 2), dtype=torch.uint8, device="cuda")
        s = torch.empty((M, d // 32), dtype=torch.uint8, device="cuda")
        mats16 = kq.kq_expand_blocks(pd, dtype=torch.bfloat16)
        extra = {}
        for log2n in (4, 6, 7):
            if d % max(32, 1 << log2n) == 0:
                pn = torch.from_numpy(inputs.lu_params(d >> log2n, seed=[M, d, 1 << log2n], factors=log2n)).cuda()
                extra[log2n] = (kq.kq_expand_blocks(pn), kq.kq_expand_factored(pn))

        def calls(xd):
            c = {
                "kroquant": lambda st: lib.kq_quantize(xd.data_ptr(), M, d, d, mats.data_ptr(), 0, fac.data_ptr(),
                                                       q.data_ptr(), s.data_ptr(), 2, 0, st),
                "kroquant_mma": lambda st: lib.kq_quantize(xd.data_ptr(), M, d, d, mats.data_ptr(), 0, None,
                                                           q.data_ptr(), s.data_ptr(), 1, 0, st),
                "kroquant_mma_bf16": lambda st: lib.kq_quantize(xd.data_ptr(), M, d, d, mats16.data_ptr(), 1, None,
                                                                q.data_ptr(), s.data_ptr(), 1, 0, st),
                "smooth": lambda st: lib.kq_ref_smooth_quantize(xd.data_ptr(), M, d, d, inv_s.data_ptr(),
                                                                q.data_ptr(), s.data_ptr(), st),
                "fwht": lambda st: lib.kq_ref_fwht_quantize(xd.data_ptr(), M, d, d, q.data_ptr(), s.data_ptr(), st),
            }
            for log2n, (mn, fn) in extra.items():
                c[f"kroquant{1 << log2n}"] = (lambda mn, fn, log2n: lambda st: lib.kq_quantize_n(
                    xd.data_ptr(), M, d, d, log2n, mn.data_ptr(), 0, fn.data_ptr(), q.data_ptr(), s.data_ptr(),
                    2, 0, st))(mn, fn, log2n)
            return c

        per_copy = [calls(xd) for xd in xs]
        reps = 60 if M * d < 2**24 else (30 if M * d < 2**28 else 10)
        res = {}
        for kind in per_copy[0]:
            fns = [pc[kind] for pc in per_copy]
            for i in range(3):
                assert fns[i % ncopy](stream) == 0
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for i in range(reps):
                assert fns[i % ncopy](stream) == 0
            b.record()
            b.synchronize()
            us = a.elapsed_time(b) * 1e3 / reps
            res[kind] = {"us": round(us, 3), "gbs": round(algo_bytes(M, d) / (us * 1e-6) / 1e9, 1)}
            if M <= 256:
                # launch-latency-bound shapes: back-to-back launches replayed from a CUDA graph
                res[kind]["graph_us_per_launch"] = round(graph_time(torch, fns[0], 50), 3)
        best_f32 = min(("kroquant", "kroquant_mma"), key=lambda k: res[k]["us"])
        line = {"sweep": name, "M": M, "d": d, "bytes": algo_bytes(M, d), "input_copies": ncopy, "launches": reps,
                **res, "best_f32_variant": best_f32,
                "kroquant_vs_smooth_speed": round(res["smooth"]["us"] / res["kroquant"]["us"], 3),
                "kroquant_vs_fwht_speed": round(res["fwht"]["us"] / res["kroquant"]["us"], 3)}
        print(json.dumps(line), flush=True)
        del xs, x0, q, s
        torch.cuda.empty_cache()
    assert kq.kq_get_device_error(clear=True) == 0


def run_profile(args) -> None:
    """Small fixed launch sequence for ncu: every kernel kind on both FLUX
    shapes, `--steps` times each, no soak, no clocks, no host-buffer pass."""
    import torch

    import mxfp4_activations_b200 as kq
    from mxfp4_activations_b200 import build

    build.build()
    kq.load()
    xs, ps = zip(*(inputs.config_case("flux", d) for d in FLUX_DS))
    step = QuantStep(torch, kq, list(xs), list(ps), n_copies=1, device=torch.device("cuda", 0))
    kinds = args.profile_kinds.split(",")
    launches = 0
    for kind in kinds:
        if kind.startswith("gemm"):
            # gemm or gemm:<shape name>: the W4A4 product on random operands
            names = [kind.split(":", 1)[1]] if ":" in kind else list(inputs.GEMM_SHAPES)
            for name in names:
                M, N, K = inputs.GEMM_SHAPES[name]
                aq, _ = inputs.mx_operand(M, K, seed=1)
                bq, _ = inputs.mx_operand(N, K, seed=2)
                sa = torch.full((kq.scale_bytes(M, K, "mma"),), 127, dtype=torch.uint8, device="cuda")
                sb = torch.full((kq.scale_bytes(N, K, "mma"),), 127, dtype=torch.uint8, device="cuda")
                a, b = torch.from_numpy(aq).cuda(), torch.from_numpy(bq).cuda()
                c = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
                for it in range(args.steps):
                    kq.kq_gemm_mxf4(a, sa, b, sb, out=c)
                    launches += 1
            continue
        for it in range(args.steps):
            for item in step.items:
                step.launch(it, item, kind)
                launches += 1
    torch.cuda.synchronize()
    assert kq.kq_get_device_error(clear=True) == 0
    print(json.dumps({"profile": kinds, "launches": launches}))


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["kq", "reference"], default="kq")
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--profile", action="store_true", help="short launch sequence for ncu")
    ap.add_argument("--profile-kinds", default="kroquant,smooth,fwht")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    elif args.profile:
        run_profile(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()

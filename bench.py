"""Benchmark: SwiGLU MLP block (d=4096, ffn=14336, Llama-3.1-8B shapes) run
through the direct-palette reconstructive GEMM on B200.

One step = one forward pass of the block at a token batch: the gate GEMM,
the up GEMM with SiLU(g)*u fused into its epilogue, and the down GEMM, all
three reading compressed weights (sign+mantissa bytes, 4-bit palette indices,
verbatim rows) and rebuilding BF16 on chip.  Synthetic N(0, 0.02) weights with
1e-4 outliers x100 stand in for Llama-3.1-8B's MLP weights.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--batch B]
    python bench.py --impl reference     # the CPU oracle on a bounded sample

Prints one JSON line on rank 0.  Multi-GPU runs (torchrun) are independent
replicas: the block does not shard on this path, so there is no collective in
the data path; the timing is the max over ranks.
"""
from __future__ import annotations

import argparse
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

METRIC = "reconstructive MLP GEMM tokens/s & effective weight GB/s vs HBM roofline, B=1–256"
D_MODEL, FFN = 4096, 14336
SIGMA, OUTLIER_RATE, OUTLIER_SCALE, SEED = 0.02, 1e-4, 100.0, 2
HBM_FALLBACK_GBS = 6650.0

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch
# of the direct-palette GEMM kernel (the 14336x4096 gate projection at batch 8,
# from one ncu --set full capture), valid only for the kernel sources it was
# taken on: reported as null once they change.
NCU_TRAFFIC = {"bytes_per_launch": 93138432,
               "launch": "gate projection 14336x4096, batch 8",
               "sources_sha256": "a5bdf8ee8d2dfb0555b9467461994f2af2809ddf6800c3e2ccae97fbc4bcd118"}
GEMM_SOURCES = ["mlp_huffman_coded_b200/csrc/uw_gemm.cu", "mlp_huffman_coded_b200/csrc/uw_device.cuh",
                "mlp_huffman_coded_b200/csrc/uw_internal.h"]


def ncu_traffic_per_launch():
    import hashlib
    h = hashlib.sha256()
    try:
        for f in GEMM_SOURCES:
            with open(os.path.join(ROOT, f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    return NCU_TRAFFIC["bytes_per_launch"] if h.hexdigest() == NCU_TRAFFIC["sources_sha256"] else None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": HBM_FALLBACK_GBS, "bf16_tflops": 1590.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 50 ms in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return self

        def reader():
            for line in self.proc.stdout:
                self.samples.append((time.time(), line.strip()))
        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()
        return self

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        rows = []
        for ts, line in self.samples:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append((ts, parts))
        inside = [r for r in rows if t0 <= r[0] <= t1]
        window = "timed region"
        if not inside:
            inside = rows
            window = "whole run (timed region shorter than the 50 ms sampling interval)"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "window": "unavailable"}
        sm = [float(p[1]) for _, p in inside if p[1].replace(".", "").isdigit()]
        smax = [float(p[2]) for _, p in inside if p[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, p in inside for i in range(4) if p[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(inside), "window": window}


def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl" if os.environ.get("UW_BENCH_BACKEND", "nccl") == "nccl" else "gloo",
                                timeout=timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _reduce_over_ranks(world, v: float, op) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    # NCCL reduces device tensors; gloo (CPU tests) host tensors
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(world, v: float) -> float:
    import torch.distributed as dist
    return _reduce_over_ranks(world, v, dist.ReduceOp.MAX)


def sum_over_ranks(world, v: float) -> float:
    import torch.distributed as dist
    return _reduce_over_ranks(world, v, dist.ReduceOp.SUM)


# ---------------------------------------------------------------------------
# CPU oracle leg (the reported CPU baseline and the --impl reference arm)
# ---------------------------------------------------------------------------

_ORACLE_PREP = {}


def oracle_prepare(batch: int, row_fraction: float):
    """Untimed preparation of the CPU sample: the first `row_fraction` of the
    rows of gate, up and down in the direct-palette form (oracle encoder and
    transcode), plus inputs of the right widths."""
    key = (batch, row_fraction)
    if key not in _ORACLE_PREP:
        from mlp_huffman_coded_b200 import synth
        from oracle import uw_oracle as O
        mats = synth.mlp_block(D_MODEL, FFN, SIGMA, OUTLIER_RATE, OUTLIER_SCALE, SEED)
        preps = []
        for w in mats:
            n = max(128, int(round(w.shape[0] * row_fraction / 128)) * 128)
            enc = O.encode(np.ascontiguousarray(w[:n]))
            preps.append((enc, O.transcode_palette(enc, lockstep=True), n / w.shape[0]))
        xs = [synth.activations(batch, D_MODEL, 3), synth.activations(batch, D_MODEL, 3),
              synth.activations(batch, FFN, 4)]
        _ORACLE_PREP[key] = (preps, xs)
    return _ORACLE_PREP[key]


def oracle_block_sample(batch: int, row_fraction: float):
    """Oracle work for one step on a row sample of each matrix: rebuild W from
    the direct-palette form (sm + 4-bit indices + verbatim rows), float64
    GEMM, SiLU(g) * u.  Returns (measured seconds, seconds scaled to the
    whole block)."""
    from oracle import uw_oracle as O
    preps, xs = oracle_prepare(batch, row_fraction)
    t0 = time.perf_counter()
    outs = []
    for (enc, idx4, _), x in zip(preps, xs):
        outs.append(O.gemm(O.rebuild_from_idx4(enc, idx4), x))
    _ = O.silu(outs[0]) * outs[1]
    dt = time.perf_counter() - t0
    frac = sum(f for _, _, f in preps) / 3
    return dt, dt / frac


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    from threadpoolctl import threadpool_limits
    frac = args.ref_fraction
    with threadpool_limits(limits=1):
        oracle_prepare(args.batch, frac)
        for _ in range(args.warmup):
            oracle_block_sample(args.batch, frac)
        times = [oracle_block_sample(args.batch, frac) for _ in range(args.steps)]
    sample_s = sum(t for t, _ in times) / len(times)     # measured seconds per (sample) step
    full_s = sum(f for _, f in times) / len(times)       # the same scaled to the whole block
    value = args.batch / full_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sample_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(args, world),
        "ms_per_step_is": "measured time of one sample step (the rows below); value uses the full block",
        "full_block_ms_per_step_extrapolated": full_s * 1e3,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: the first {frac:.4f} of the rows of gate, up and down "
                                   f"(direct-palette rebuild + float64 GEMM + SiLU*up); tokens/s from its time "
                                   f"scaled by the rows covered to the full block"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(args, world: int = 1):
    """The workload, identical for the GPU arm and the oracle arm."""
    return {"workload": f"SwiGLU MLP block d={D_MODEL} ffn={FFN} (Llama-3.1-8B shapes), direct-palette "
                        f"reconstructive GEMM, batch {args.batch}",
            "batch": args.batch, "d_model": D_MODEL, "ffn": FFN, "pipeline": "direct palette (gate, up, down)",
            "weights": f"N(0,{SIGMA}) bf16, outliers {OUTLIER_RATE} x{OUTLIER_SCALE}, seed {SEED}",
            "l2": "inputs larger than L2: 3 compressed matrices (~268 MB) streamed per step, L2 is 126 MB",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_gpu(args, world, rank, local):
    import torch
    from mlp_huffman_coded_b200 import synth, uw

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B = args.batch
    mats = synth.mlp_block(D_MODEL, FFN, SIGMA, OUTLIER_RATE, OUTLIER_SCALE, SEED)
    encs = [uw.encode(w) for w in mats]
    dms = []
    ws0 = uw.Workspace(256, device=dev)
    for e in encs:
        dms.append(uw.DeviceMatrix(e, device=dev).prepare_direct_palette(ws0))
    ws0.check("load-time transcode")
    pipes = [uw.PIPE_DIRECT] * 3
    ws = uw.Workspace(uw.mlp_workspace_bytes(*dms, pipes, B), device=dev)
    x_host = synth.activations(B, D_MODEL, 3)
    x = torch.from_numpy(x_host.view(np.int16)).to(dev)
    y = torch.empty(B, D_MODEL, dtype=torch.int16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        uw.mlp_block(*dms, pipes, x, y, ws, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    ws.check("warmup")

    sampler = ClockSampler(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[0])
                           if os.environ.get("CUDA_VISIBLE_DEVICES", "").replace(",", "").isdigit() else local)
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    launches0 = uw.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    e1.synchronize()
    t_wall1 = time.time()
    torch.cuda.synchronize(dev)
    barrier(world)
    launches = uw.launch_count() - launches0
    ms = e0.elapsed_time(e1)
    ms = max_over_ranks(world, ms)
    ws.check("timed region")
    time.sleep(0.3)
    sampler.stop()
    clocks = sampler.summary(t_wall0 - 0.05, t_wall1 + 0.05)

    # end to end: every step copies its x from pinned host memory to the
    # device, runs the block and copies its y back to pinned host memory.
    # The copies run on their own streams with double-buffered device x / y,
    # so step i+1's input copy and step i's output copy overlap the blocks
    # around them (events order each copy after the compute it depends on).
    x_pin = torch.from_numpy(x_host.view(np.int16)).pin_memory()
    y_pin = [torch.empty(B, D_MODEL, dtype=torch.int16).pin_memory() for _ in range(2)]
    x_e = [torch.empty_like(x) for _ in range(2)]
    y_e = [torch.empty_like(y) for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    x_in = [torch.cuda.Event() for _ in range(2)]     # x_e[b] holds its step's input
    done = [torch.cuda.Event() for _ in range(2)]     # the block of buffer b finished
    y_out = [torch.cuda.Event() for _ in range(2)]    # y_e[b] has been read back

    def e2e_steps(n):
        for i in range(n):
            b = i & 1
            if i >= 2:
                h2d.wait_event(done[b])                # step i-2 no longer reads x_e[b]
            with torch.cuda.stream(h2d):
                x_e[b].copy_(x_pin, non_blocking=True)
                x_in[b].record(h2d)
            stream.wait_event(x_in[b])
            if i >= 2:
                stream.wait_event(y_out[b])            # step i-2's y has left y_e[b]
            uw.mlp_block(*dms, pipes, x_e[b], y_e[b], ws, stream)
            done[b].record(stream)
            d2h.wait_event(done[b])
            with torch.cuda.stream(d2h):
                y_pin[b].copy_(y_e[b], non_blocking=True)
                y_out[b].record(d2h)
        stream.wait_stream(h2d)
        stream.wait_stream(d2h)

    e2e_steps(4)
    torch.cuda.synchronize(dev)
    barrier(world)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    h2d.wait_stream(stream)   # no copy of the timed steps starts before f0
    d2h.wait_stream(stream)
    e2e_steps(args.steps)
    f1.record(stream)
    f1.synchronize()
    e2e_ms = max_over_ranks(world, f0.elapsed_time(f1))
    assert torch.equal(y_pin[(args.steps - 1) & 1], y.cpu()), "end-to-end output differs from the resident run"

    # uncompressed BF16 comparator (cuBLAS through torch.matmul) on the same shapes
    wt = [torch.from_numpy(w.view(np.int16)).to(dev).view(torch.bfloat16) for w in mats]
    xb = x.view(torch.bfloat16)

    def step_bf16():
        g = xb @ wt[0].T
        u = xb @ wt[1].T
        h = torch.nn.functional.silu(g) * u
        return h @ wt[2].T

    for _ in range(3):
        step_bf16()
    torch.cuda.synchronize(dev)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(args.steps):
        step_bf16()
    g1.record(stream)
    g1.synchronize()
    bf16_ms = g0.elapsed_time(g1) / args.steps
    del wt

    # roofline of the dominant kernel (the reconstructive GEMM: every launch of
    # the step is one)
    peaks, src = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    w_bytes = sum(dm.direct_palette_bytes() for dm in dms)

    def step_bytes(b):
        return w_bytes + 2 * b * (D_MODEL + FFN) * 2 + 2 * b * FFN * 2

    per_step_bytes = step_bytes(B)
    t_step = ms / 1e3 / args.steps
    # a step is 3 launches of the GEMM kernel back to back (gate, up with the
    # fused SwiGLU, down); they tile the step, so the average launch lasts a
    # third of it and moves a third of its algorithmic bytes
    launch_s = t_step / 3
    bytes_per_launch = per_step_bytes / 3
    achieved = bytes_per_launch / launch_s / 1e9

    # the gate launch alone, timed launch by launch with CUDA events on the
    # launching stream, L2 flushed before each (outside the timed interval)
    flush = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
    ws_g = uw.Workspace(uw.workspace_bytes(dms[0], uw.PIPE_DIRECT, B), device=dev)
    g_out = torch.empty(B, FFN, dtype=torch.int16, device=dev)
    iso = []
    for i in range(args.warmup + 20):
        flush.view(torch.int32).max()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        uw.gemm_direct_palette(dms[0], x, g_out, ws_g, stream)
        a1.record(stream)
        a1.synchronize()
        if i >= args.warmup:
            iso.append(a0.elapsed_time(a1) / 1e3)
    ws_g.check("gate launch")
    iso_s = float(np.median(iso))
    gate_bytes = dms[0].direct_palette_bytes() + 2 * B * (D_MODEL + FFN)
    del ws_g, g_out, flush

    # the other batches the block is quoted at (1 and 32 next to the default
    # 8): the same step, timed the same way, plus the BF16 comparator
    other = {}
    for b in [v for v in (1, 8, 32) if v != B]:
        wsb = uw.Workspace(uw.mlp_workspace_bytes(*dms, pipes, b), device=dev)
        xb_dev = torch.from_numpy(synth.activations(b, D_MODEL, 3).view(np.int16)).to(dev)
        yb_dev = torch.empty(b, D_MODEL, dtype=torch.int16, device=dev)
        for _ in range(args.warmup):
            uw.mlp_block(*dms, pipes, xb_dev, yb_dev, wsb, stream)
        torch.cuda.synchronize(dev)
        n_b = max(3, args.steps)
        h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h0.record(stream)
        for _ in range(n_b):
            uw.mlp_block(*dms, pipes, xb_dev, yb_dev, wsb, stream)
        h1.record(stream)
        h1.synchronize()
        wsb.check(f"batch {b}")
        ms_b = max_over_ranks(world, h0.elapsed_time(h1)) / n_b
        wt_b = [torch.from_numpy(w.view(np.int16)).to(dev).view(torch.bfloat16) for w in mats]
        xbb = xb_dev.view(torch.bfloat16)

        def step_bf16_b():
            g = xbb @ wt_b[0].T
            u = xbb @ wt_b[1].T
            return (torch.nn.functional.silu(g) * u) @ wt_b[2].T

        for _ in range(3):
            step_bf16_b()
        torch.cuda.synchronize(dev)
        h0.record(stream)
        for _ in range(n_b):
            step_bf16_b()
        h1.record(stream)
        h1.synchronize()
        bf16_b = h0.elapsed_time(h1) / n_b
        del wt_b
        ach_b = step_bytes(b) / (ms_b / 1e3) / 1e9
        other[str(b)] = {"ms_per_step": ms_b, "tokens_per_s": b * world / (ms_b / 1e3), "steps": n_b,
                         "roofline_frac": ach_b / peak, "achieved_gbs": ach_b,
                         "bf16_torch_matmul_ms_per_step": bf16_b, "speedup_vs_bf16_torch": bf16_b / ms_b}
    weight_gbs = sum(2 * e.rows * e.cols for e in encs) / t_step / 1e9

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": B * args.steps * world / (ms / 1e3),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms / args.steps,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": config_dict(args, world),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": ncu_traffic_per_launch(),
                         "traffic_launch": NCU_TRAFFIC["launch"],
                         "kernel": "gemm_kernel<PACK, uniform palette> (direct-palette reconstructive GEMM)",
                         "launches_per_step": 3, "avg_launch_us": launch_s * 1e6,
                         "algorithmic_bytes_per_launch": bytes_per_launch,
                         "algorithmic_bytes_per_step": per_step_bytes,
                         "isolated_gate_launch": {"us": iso_s * 1e6, "algorithmic_bytes": gate_bytes,
                                                  "achieved_gbs": gate_bytes / iso_s / 1e9,
                                                  "frac": gate_bytes / iso_s / 1e9 / peak,
                                                  "timing": "median of 20 launches, CUDA events on the launching "
                                                            "stream, L2 flushed before each"},
                         "peak_source": f"{src} hbm_gbs ({'of measured' if src == 'measured' else 'of fallback'})"},
            "effective_weight_gbs": weight_gbs,
            "other_batches": other,
            "bf16_torch_matmul_ms_per_step": bf16_ms,
            "speedup_vs_bf16_torch": bf16_ms / (ms / args.steps),
            "e2e": {"value": B * args.steps * world / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": B * D_MODEL * 2, "d2h_bytes_per_step": B * D_MODEL * 2},
            "gpu_launches": int(launches),
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                oracle_prepare(B, args.ref_fraction)
                dt = min(oracle_block_sample(B, args.ref_fraction)[1] for _ in range(3))
            line["cpu_baseline"] = {
                "value": B / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                "sample": f"best of 3 steps on {args.ref_fraction:.4f} of the rows of gate, up and down "
                          f"(direct-palette rebuild + float64 GEMM), scaled to the full block; "
                          f"os.cpu_count()={os.cpu_count()}"}
        print(json.dumps(line), flush=True)
    return 0


def run_gemm_case(args, local):
    """One matrix (gate, 14336x4096) through one pipeline: the unit that ncu
    captures of the GEMM are taken on.  Prints a small JSON line."""
    import torch
    from mlp_huffman_coded_b200 import synth, uw
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = synth.mlp_block(D_MODEL, FFN, SIGMA, OUTLIER_RATE, OUTLIER_SCALE, SEED)[0]
    enc = uw.encode(w)
    dm = uw.DeviceMatrix(enc, device=dev)
    ws = uw.Workspace(max(uw.workspace_bytes(dm, p, args.batch) for p in range(4)), device=dev)
    dm.prepare_direct_palette(ws)
    x = torch.from_numpy(synth.activations(args.batch, D_MODEL, 3).view(np.int16)).to(dev)
    y = torch.empty(args.batch, FFN, dtype=torch.int16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    if args.pipeline == "bf16":
        wd = torch.from_numpy(w.view(np.int16)).to(dev)
        ws = uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_BF16, args.batch), device=dev)

        def call():
            uw.gemm_bf16(wd, x, y, ws)
    else:
        pipe = uw.PIPELINES[args.pipeline]

        def call():
            uw.gemm(dm, pipe, x, y, ws)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    times = []
    flush.fill_(1)
    for _ in range(args.steps):
        if not args.no_flush:
            # read (not write) a buffer larger than L2, so L2 holds clean
            # lines and the timed call pays no write-backs
            flush.view(torch.int32).max()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    ws.check("gemm case")
    t = float(np.median(times))
    nbytes = dm.direct_palette_bytes() if args.pipeline == "direct" else None
    print(json.dumps({"case": "gemm", "pipeline": args.pipeline, "batch": args.batch, "median_us": t,
                      "min_us": float(np.min(times)), "direct_bytes": nbytes,
                      "gbs": (nbytes / t / 1e3) if nbytes else None}), flush=True)
    return 0


def _timed(call, flush, steps, warmup, dev):
    """Median / min µs of `call` over `steps` runs, L2 flushed (clean read of a
    256 MB buffer) before each, CUDA events on the current stream."""
    import torch
    for _ in range(warmup):
        call()
    torch.cuda.synchronize(dev)
    times = []
    for _ in range(steps):
        flush.view(torch.int32).max()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    return float(np.median(times)), float(np.min(times))


def run_decode_case(args, local):
    """The three preprocessing decoders on the 14336x4096 gate-shaped matrix
    (sigma 0.02, 1e-4 outliers x100, seed 1): µs, GB/s of compressed input
    read and of output written, and (read + write) / time against HBM."""
    import torch
    from mlp_huffman_coded_b200 import synth, uw
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = synth.weight_matrix(FFN, D_MODEL, SIGMA, OUTLIER_RATE, OUTLIER_SCALE, seed=1)
    enc = uw.encode(w)
    dm = uw.DeviceMatrix(enc, device=dev)
    ws = uw.Workspace(256, device=dev)
    flush = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
    n = w.size
    meta = enc.chunk_bit_off.nbytes + enc.vflags.nbytes + enc.vprefix.nbytes
    stream = enc.stream.nbytes
    verb = enc.verbatim.nbytes
    peaks, src = measured_peaks()
    hbm = peaks.get("hbm_gbs", HBM_FALLBACK_GBS)
    cases = [
        ("full", torch.empty(n, dtype=torch.int16, device=dev), uw.decode_full, enc.sm.nbytes + stream + meta + verb, 2 * n),
        ("exponent", torch.empty(n, dtype=torch.uint8, device=dev), uw.decode_exponent_only, stream + meta + verb, n),
        ("transcode", torch.empty(n // 2, dtype=torch.uint8, device=dev), uw.transcode_palette, stream + meta, n // 2),
    ]
    for name, out, fn, rd, wr in cases:
        med, mn = _timed(lambda: fn(dm, out, ws), flush, args.steps, args.warmup, dev)
        ws.check(f"decode {name}")
        print(json.dumps({"case": "decode", "decoder": name, "matrix": "14336x4096 seed 1", "median_us": med,
                          "min_us": mn, "read_bytes": rd, "write_bytes": wr, "read_gbs": rd / med / 1e3,
                          "write_gbs": wr / med / 1e3, "hbm_frac": (rd + wr) / med / 1e3 / hbm,
                          "hbm_peak_gbs": hbm, "peak_source": src}), flush=True)
    return 0


def run_sweep_case(args, local):
    """SwiGLU block matrices x batch 1..512: the four pipelines, the library's
    own BF16 GEMM and torch.matmul BF16 (cuBLAS), L2 flushed before each call;
    then the autotuner's choice per matrix and batch."""
    import torch
    from mlp_huffman_coded_b200 import synth, uw
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    batches = [1, 2, 4, 8, 16, 32, 64, 128, 256, 512]
    mats = synth.mlp_block(D_MODEL, FFN, SIGMA, OUTLIER_RATE, OUTLIER_SCALE, SEED)
    names = ["gate", "up", "down"]
    flush = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
    ws0 = uw.Workspace(256, device=dev)
    for name, w in zip(names, mats):
        dm = uw.DeviceMatrix(uw.encode(w), device=dev).prepare_direct_palette(ws0)
        ws0.check("prepare")
        N, K = w.shape
        wd = torch.from_numpy(w.view(np.int16)).to(dev)
        wt = wd.view(torch.bfloat16)
        ws = uw.Workspace(max(max(uw.workspace_bytes(dm, p, max(batches)) for p in range(4)),
                              uw.workspace_bytes(dm, uw.PIPE_BF16, max(batches))), device=dev)
        xall = torch.from_numpy(synth.activations(max(batches), K, 3).view(np.int16)).to(dev)
        for B in batches:
            x = xall[:B].contiguous()
            y = torch.empty(B, N, dtype=torch.int16, device=dev)
            row = {"case": "sweep", "matrix": f"{name} {N}x{K}", "batch": B}
            for pname, pipe in (("full", uw.PIPE_FULL), ("exponent", uw.PIPE_EXPONENT),
                                ("transcode", uw.PIPE_TRANSCODE), ("direct", uw.PIPE_DIRECT)):
                row[pname + "_us"] = _timed(lambda: uw.gemm(dm, pipe, x, y, ws), flush, args.steps, args.warmup, dev)[0]
            row["own_bf16_us"] = _timed(lambda: uw.gemm_bf16(wd, x, y, ws), flush, args.steps, args.warmup, dev)[0]
            xb = x.view(torch.bfloat16)
            row["torch_bf16_us"] = _timed(lambda: xb @ wt.T, flush, args.steps, args.warmup, dev)[0]
            ws.check("sweep")
            print(json.dumps(row), flush=True)
        y = torch.empty(max(batches), N, dtype=torch.int16, device=dev)
        choice, us = uw.autotune(dm, batches, max(3, args.steps // 2), xall, y, ws, flush=flush)
        ws.check("autotune")
        print(json.dumps({"case": "autotune", "matrix": f"{name} {N}x{K}", "batches": batches,
                          "choice": [["full", "exponent", "transcode", "direct"][c] for c in choice],
                          "us": np.round(us, 2).tolist()}), flush=True)
        del dm, wd, ws
        torch.cuda.empty_cache()
    return 0


def run_stack_case(args):
    """Compressed size of the 32-layer MLP stack (96 matrices, per-layer sigma
    uniform in [0.01, 0.05], 1e-3 outliers x100): host encoder only, no GPU."""
    from mlp_huffman_coded_b200 import synth, uw
    n_layers = args.layers
    tot = dict(bf16=0, huffman=0, pack=0, verbatim=0, groups=0, bits=0, coded=0)
    for layer in range(n_layers):
        for name, w in zip(("gate", "up", "down"), synth.stack_layer(layer)):
            e = uw.encode(w)
            _, pack = e.pack_offsets()
            nv, ng = int(e.layout.n_verbatim), int(e.layout.n_groups)
            bits = int(e.chunk_bit_off[-1])
            tot["bf16"] += w.nbytes
            tot["huffman"] += e.compressed_bytes("huffman")
            tot["pack"] += pack
            tot["verbatim"] += nv
            tot["groups"] += ng
            tot["bits"] += bits
            tot["coded"] += (ng - nv) * 64
            print(json.dumps({"case": "stack", "layer": layer, "matrix": name,
                              "sigma": round(float(synth.stack_sigmas()[layer]), 5), "bf16_bytes": w.nbytes,
                              "huffman_ratio": e.compressed_bytes("huffman") / w.nbytes,
                              "pack_ratio": pack / w.nbytes, "verbatim_frac": nv / ng,
                              "mean_code_bits": bits / max(1, (ng - nv) * 64)}), flush=True)
    print(json.dumps({"case": "stack", "layers": n_layers, "matrices": 3 * n_layers,
                      "bf16_gb": tot["bf16"] / 1e9, "huffman_gb": tot["huffman"] / 1e9,
                      "huffman_ratio": tot["huffman"] / tot["bf16"], "pack_gb": tot["pack"] / 1e9,
                      "pack_ratio": tot["pack"] / tot["bf16"], "verbatim_frac": tot["verbatim"] / tot["groups"],
                      "mean_code_bits": tot["bits"] / max(1, tot["coded"])}), flush=True)
    return 0


def run_stack_time_case(args, local):
    """Per-decode-step MLP time of the whole stack (default 32 layers = 96
    matrices, per-layer sigma uniform in [0.01, 0.05], 1e-3 outliers x100) at
    batch 1 and 64, measured end to end: every layer's weights are drawn on
    the GPU (synth.stack_layer_device: the stack recipe with torch's
    generator), compressed and packed on the GPU, each matrix's pipeline is
    picked by uw_autotune, and one timed step is one uw_mlp_stack call (all
    GEMMs of all layers, back to back on one stream).  L2 is flushed before
    each step (the packed stack is ~9 GB anyway).  Beside it: the same
    layers in BF16 through torch (cuBLAS matmul, SiLU * up), weights
    resident, timed the same way."""
    import torch
    import torch.nn.functional as F
    from mlp_huffman_coded_b200 import synth, uw
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    n_layers = args.layers
    batches = [1, 64]
    flush = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
    ws0 = uw.Workspace(256, device=dev)
    layers, bf16, choices = [], [], []
    pack_bytes = 0
    t0 = time.time()
    xa = ya = None
    for layer in range(n_layers):
        ws_bf16 = synth.stack_layer_device(layer, dev)
        triple, ch = [], []
        for w in ws_bf16:
            dm = uw.DeviceMatrix.encode_on_device(w).prepare_direct_palette(ws0, keep_idx4=False)
            ws0.check("prepare")
            rows, cols = int(dm.mat.L.rows), int(dm.mat.L.cols)
            if xa is None or xa.shape[1] < cols or ya.shape[1] < rows:
                xa = torch.from_numpy(synth.activations(max(batches), max(cols, 14336), 3).view(np.int16)).to(dev)
                ya = torch.empty(max(batches), max(rows, 14336), dtype=torch.int16, device=dev)
            wsa = uw.Workspace(max(uw.workspace_bytes(dm, p, max(batches)) for p in range(4)), device=dev)
            c, _ = uw.autotune(dm, batches, 3, xa[:, :cols].contiguous(), ya, wsa, flush=flush)
            wsa.check("autotune")
            del wsa
            pack_bytes += dm.direct_palette_bytes()
            triple.append(dm)
            ch.append([int(v) for v in c])
        layers.append(triple)
        choices.append(ch)
        bf16.append(tuple(w.view(torch.bfloat16) for w in ws_bf16))
    prep_s = time.time() - t0
    d = int(layers[0][0].mat.L.cols)
    for bi, B in enumerate(batches):
        pipes = [[ch[j][bi] for j in range(3)] for ch in choices]
        ws = uw.Workspace(uw.mlp_stack_workspace_bytes(layers, pipes, B), device=dev)
        x = torch.from_numpy(synth.activations(B, d, 3).view(np.int16)).to(dev)
        y = torch.empty(B, d, dtype=torch.int16, device=dev)
        med, mn = _timed(lambda: uw.mlp_stack(layers, pipes, x, y, ws), flush, args.steps, args.warmup, dev)
        ws.check("stack")
        xb = x.view(torch.bfloat16)

        def torch_stack():
            h = xb
            for g, u, dn in bf16:
                h = (F.silu(h @ g.T) * (h @ u.T)) @ dn.T
            return h
        tmed, tmn = _timed(torch_stack, flush, args.steps, args.warmup, dev)
        used = sorted({uw.PIPE_NAMES[p] for triple in pipes for p in triple})
        print(json.dumps({"case": "stack-time", "layers": n_layers, "matrices": 3 * n_layers, "batch": B,
                          "step_ms": med / 1e3, "step_ms_min": mn / 1e3, "tokens_per_s": B / (med / 1e6),
                          "packed_gb": pack_bytes / 1e9,
                          "packed_gbs": pack_bytes / (med / 1e6) / 1e9,
                          "torch_bf16_step_ms": tmed / 1e3,
                          "speedup_vs_bf16_torch": tmed / med,
                          "pipelines_used": used, "launch": "one uw_mlp_stack call per step",
                          "weights": "drawn on the GPU (torch generator, stack recipe)",
                          "prep_s": round(prep_s, 1)}), flush=True)
        del ws
    return 0


def run_shapes_case(args, local):
    """The scheme on the non-MLP matrices of a Llama-3.1-8B-shaped model
    (weights drawn on the GPU with the MLP recipe: N(0, 0.02), 1e-4
    outliers x100; compressed on the GPU): direct-palette GEMM vs
    torch.matmul BF16 for q/o (4096 x 4096), k/v (1024 x 4096) and the
    output projection (128256 x 4096) at batch 1, 8, 64, L2 flushed before
    each call; and the embedding lookup of 64 tokens from a compressed
    128256 x 4096 table (uw_decode_rows) vs torch.index_select on BF16."""
    import torch
    from mlp_huffman_coded_b200 import synth, uw
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    flush = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
    ws0 = uw.Workspace(256, device=dev)
    peaks, src = measured_peaks()
    hbm = peaks.get("hbm_gbs", HBM_FALLBACK_GBS)
    shapes = [("q_proj/o_proj", 4096, 4096, 130), ("k_proj/v_proj", 1024, 4096, 131),
              ("lm_head", 128256, 4096, 132)]
    for name, rows, cols, seed in shapes:
        w = synth.weight_matrix_device(rows, cols, SIGMA, OUTLIER_RATE, OUTLIER_SCALE, seed, dev)
        dm = uw.DeviceMatrix.encode_on_device(w).prepare_direct_palette(ws0, keep_idx4=False)
        ws0.check("prepare")
        wb = w.view(torch.bfloat16)
        for B in (1, 8, 64):
            x = torch.from_numpy(synth.activations(B, cols, 3).view(np.int16)).to(dev)
            y = torch.empty(B, rows, dtype=torch.int16, device=dev)
            ws = uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_DIRECT, B), device=dev)
            med, _ = _timed(lambda: uw.gemm_direct_palette(dm, x, y, ws), flush, args.steps, args.warmup, dev)
            ws.check("gemm")
            xb = x.view(torch.bfloat16)
            tmed, _ = _timed(lambda: xb @ wb.T, flush, args.steps, args.warmup, dev)
            nbytes = dm.direct_palette_bytes()
            print(json.dumps({"case": "shapes", "matrix": f"{name} {rows}x{cols}", "batch": B,
                              "direct_palette_us": med, "torch_bf16_us": tmed, "speedup_vs_bf16": tmed / med,
                              "packed_bytes": nbytes, "bf16_bytes": rows * cols * 2,
                              "packed_gbs": nbytes / med / 1e3, "hbm_frac": nbytes / med / 1e3 / hbm,
                              "hbm_peak_gbs": hbm, "peak_source": src}), flush=True)
            del ws
        if name == "lm_head":
            ids = torch.from_numpy(np.random.default_rng(5).integers(0, rows, 64).astype(np.int32)).to(dev)
            out = torch.empty(64, cols, dtype=torch.int16, device=dev)
            med, _ = _timed(lambda: uw.decode_rows(dm, ids, out, ws0), flush, args.steps, args.warmup, dev)
            ws0.check("decode rows")
            tmed, _ = _timed(lambda: torch.index_select(wb, 0, ids), flush, args.steps, args.warmup, dev)
            print(json.dumps({"case": "shapes", "matrix": f"embedding {rows}x{cols}", "tokens": 64,
                              "decode_rows_us": med, "torch_index_select_us": tmed}), flush=True)
        del dm, w, wb
        torch.cuda.empty_cache()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 3000 GPU steps, ~0.3 s; 20 oracle samples for --impl reference)")
    ap.add_argument("--warmup", type=int, default=None, help="untimed steps (default 20; 3 for --impl reference)")
    ap.add_argument("--batch", type=int, default=8)
    ap.add_argument("--impl", default="uw", choices=["uw", "reference"])
    ap.add_argument("--ref-fraction", type=float, default=1 / 16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=32, help="stack / stack-time cases: layers to use")
    ap.add_argument("--case", default="block",
                    choices=["block", "gemm", "decode", "sweep", "stack", "stack-time", "shapes"],
                    help="gemm: one 14336x4096 matrix through --pipeline (profiling unit); decode: the three "
                         "decoders on it; sweep: pipelines x batch 1..512 x block matrices + autotune; "
                         "stack: compressed size of the 32-layer stack (host only); stack-time: decode-step "
                         "MLP time of the --layers-layer stack (one uw_mlp_stack call) at batch 1 and 64; shapes: "
                         "attention / output-projection GEMMs and the embedding lookup")
    ap.add_argument("--pipeline", default="direct", choices=["full", "exponent", "transcode", "direct", "bf16"])
    ap.add_argument("--no-flush", action="store_true", help="gemm case: leave L2 warm between calls")
    args = ap.parse_args(argv)
    if args.steps is None:
        args.steps = 20 if args.impl == "reference" else {"gemm": 100, "decode": 20, "sweep": 10,
                                                         "stack-time": 20, "shapes": 20}.get(args.case, 3000)
    if args.warmup is None:
        args.warmup = 3 if args.impl == "reference" or args.case in ("sweep", "decode", "stack-time",
                                                                       "shapes") else 20
    if args.case == "stack":
        return run_stack_case(args)
    world, rank, local = dist_init()
    try:
        if args.impl == "reference":
            return run_reference(args, world, rank)
        if args.case == "gemm":
            return run_gemm_case(args, local)
        if args.case == "decode":
            return run_decode_case(args, local)
        if args.case == "sweep":
            return run_sweep_case(args, local)
        if args.case == "stack-time":
            return run_stack_time_case(args, local)
        if args.case == "shapes":
            return run_shapes_case(args, local)
        return run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())

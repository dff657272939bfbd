#!/usr/bin/env python
"""Benchmark of the W8A8 FP8 block-scaled linear on B200.

One step = one fused linear call (fp8q_linear: per-token-group FP8
quantization of X plus the block-scaled FP8 GEMM) on one batch of
synthetic activations, at the prefill projection M=1168, K=5120, N=17408
(the up-projection shape the pages quote for act-quant GB/s and linear
TFLOP/s). Inputs are resident in HBM when the timed region starts; the
steps rotate over three input sets (X, W, Y and workspace, ~450 MB) so
no step reads what the previous one left in the 126 MB L2.

Prints ONE JSON line (rank 0). With --gpus N under torchrun each rank runs
its own replica on its own tokens (weak scaling; the path has no exchange
step), and the time is the max over ranks.

--impl reference times the CPU oracle (the plain restatement of the method
in oracle/) on a bounded sample of the same workload on the host cores.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "FP8 block-scaled linear TFLOP/s & act-quant GB/s, % of B200 roofline"
WORKLOADS = {
    "prefill_m1168_n17408_k5120": dict(m=1168, n=17408, k=5120, p=0.01, sigma=20.0, number=4),
    "prefill_m4576_n6144_k6144": dict(m=4576, n=6144, k=6144, p=0.001, sigma=50.0, number=5),
    "prefill_m4576_n6144_k17408": dict(m=4576, n=6144, k=17408, p=0.001, sigma=50.0, number=5),
    "decode_m25_n6144_k5120": dict(m=25, n=6144, k=5120, p=0.01, sigma=20.0, number=2),
    "decode_m25_n5120_k17408": dict(m=25, n=5120, k=17408, p=0.01, sigma=20.0, number=3),
}
# The dense FFN built on the same kernels (x quantized once, one gate|up
# GEMM, SiLU*up quantized for the down GEMM): D = 5120, I = 17408.
FFN_WORKLOADS = {
    "ffn_m1168_d5120_i17408": dict(m=1168, d=5120, i=17408, seed=1100),
    "ffn_m25_d5120_i17408": dict(m=25, d=5120, i=17408, seed=1100),
}
FFN_METRIC = "dense FFN (FP8 block-scaled, x quantized once) TFLOP/s"
# The NVFP4 projection arm at the FP8 path's shapes (x packed to E2M1 with
# E4M3 block scales inside the call, times a packed weight).
NVFP4_WORKLOADS = {
    "nvfp4_m1168_n17408_k5120": dict(m=1168, n=17408, k=5120, seed=1200),
    "nvfp4_m25_n6144_k5120": dict(m=25, n=6144, k=5120, seed=1201),
}
NVFP4_METRIC = "NVFP4 projection (x packed in the call) TFLOP/s"
DEFAULT_WORKLOAD = "prefill_m1168_n17408_k5120"
N_SETS = 3


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def quant_bytes(m, k, row_major=True):
    """Algorithmic HBM bytes of one fp8q_quant_act call: read X (2 B an
    element), write Q (1 B), the K-major scales with their pad rows and, as
    the call emits them, the row-major scales (4 B a group each)."""
    g = k // 128
    mp = -(-m // 16) * 16
    return 2 * m * k + m * k + 4 * g * mp + (4 * g * m if row_major else 0)


def gemm_hbm_bytes(m, n, k):
    g = k // 128
    mp = -(-m // 16) * 16
    return m * k + n * k + 4 * g * mp + 4 * (n // 128) * g + 2 * m * n


# The source files each kernel is built from; a recorded DRAM traffic figure
# stays valid while their hash is unchanged.
KERNEL_SOURCES = {
    "gemm_blockscaled_kernel": ["gemm.cu", "group_quant.cuh", "ptx.cuh", "internal.h"],
    "gemm_decode_kernel": ["gemm.cu", "group_quant.cuh", "ptx.cuh", "internal.h"],
    "quant_act_stream_kernel": ["quant.cu", "group_quant.cuh", "ptx.cuh", "internal.h"],
    "quant_act_single_kernel": ["quant.cu", "group_quant.cuh", "ptx.cuh", "internal.h"],
    "silu_mul_quant_kernel": ["ffn.cu", "group_quant.cuh", "ptx.cuh"],
}


# B200 dense FP8 tensor throughput as specified (not measured), reported
# beside the measured-bf16-based peak.
FP8_NOMINAL_TFLOPS = 4500.0


def strip_comments(src: str) -> str:
    """C/C++ source without its comments and with whitespace runs collapsed,
    so that editing a comment does not change a kernel's digest."""
    import re
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_digest(kernel: str) -> str:
    """Digest of the code (comments stripped) of a kernel's source files."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "fp8_block_scaled_group_b200", "csrc", name), encoding="utf-8") as f:
            h.update(strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def read_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded from an ncu capture in profiles/traffic.txt,
    or None when absent or when the kernel's sources changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path) or kernel not in KERNEL_SOURCES:
        return None
    digest = kernel_digest(kernel)
    with open(path) as f:
        for line in f:
            parts = line.split("#", 1)[0].split()
            if len(parts) == 4 and parts[0] == kernel and parts[1] == workload and parts[3] == digest:
                return float(parts[2])
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                smax = float(p[2])
            except ValueError:
                continue
            for nm, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int, device: str = "cuda") -> float:
    """The largest value over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device: str = "cuda") -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_input_seed(seed_base: int, rank: int, set_index: int) -> int:
    """Seed of input set `set_index` on `rank`: every rank draws its own tokens."""
    return seed_base + 7919 * (rank * N_SETS + set_index)


def weak_scaling_value(units_per_rank_step: float, world: int, steps: int, ms_total: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest
    rank's time (units per second)."""
    return units_per_rank_step * world * steps / (ms_total * 1e-3)


def hold_stream(steps: int):
    """A spin kernel ahead of timed launches keeps the GPU busy while the host
    enqueues them, so the device runs them back to back and the events
    measure device time, not host launch overhead."""
    import torch
    torch.cuda._sleep(int(2e6 + 2e5 * steps))


def stream_loop_ms(fn, steps: int) -> float:
    """Average device time per call of `steps` calls launched back to back on
    the current stream (CUDA events on that stream)."""
    import torch
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    hold_stream(steps)
    e0.record(stream)
    for i in range(steps):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def graph_loop_ms(fn, steps: int, replays: int = 5) -> float:
    """Average device time per call of `steps` calls captured in one CUDA
    graph (no host launch work between them), median over `replays` replays,
    CUDA events on the replaying stream. `fn` must have run before (set-up
    such as shared-memory opt-in happens on first calls, outside capture)."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            for i in range(steps):
                fn(i)
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    times = []
    for _ in range(replays):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / steps)
    del graph
    return statistics.median(times)


E2E_DEPTH = 2  # steps in flight in the end-to-end loop (device input/output buffers per stream)
E2E_OVERLAP = "input copy, call and result copy of consecutive steps on three streams, 2 steps in flight"


def pipelined_e2e_ms(h2d, compute, d2h, steps: int, warmup: int) -> float:
    """Device time per step of the end-to-end loop, as a server runs it: step
    i's input copy (host -> device), step i-1's call and step i-2's result copy
    (device -> host) run at once on three streams (the host link is full
    duplex), with E2E_DEPTH device buffers per direction. Every step still
    copies its own input in and its own result out. h2d(i, b), compute(i, b)
    and d2h(i, b) enqueue step i's part on the current stream, using buffer b.
    Timed with CUDA events on the calling stream, which waits for all three."""
    import torch
    cur = torch.cuda.current_stream()
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(E2E_DEPTH)]
    run_done = [torch.cuda.Event() for _ in range(E2E_DEPTH)]
    out_done = [torch.cuda.Event() for _ in range(E2E_DEPTH)]

    def run(n: int, timed: bool) -> float:
        if timed:
            hold_stream(n)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        for s in (s_in, s_run, s_out):
            s.wait_event(e0)
        for i in range(n):
            b = i % E2E_DEPTH
            with torch.cuda.stream(s_in):
                if i >= E2E_DEPTH:
                    s_in.wait_event(run_done[b])  # the call that read input buffer b is done
                h2d(i, b)
                in_done[b].record(s_in)
            with torch.cuda.stream(s_run):
                s_run.wait_event(in_done[b])
                if i >= E2E_DEPTH:
                    s_run.wait_event(out_done[b])  # output buffer b has been copied out
                compute(i, b)
                run_done[b].record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(run_done[b])
                d2h(i, b)
                out_done[b].record(s_out)
        for s in (s_in, s_run, s_out):
            cur.wait_stream(s)
        e1.record(cur)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / max(1, n)

    run(max(warmup, E2E_DEPTH + 1), False)
    return run(steps, True)


L2_BYTES = 126 * 2 ** 20


def rotation(bytes_per_set: int, lo: int = 2, hi: int = 24) -> int:
    """Input sets to rotate so that one pass over them moves more than 3x the
    L2 size: no launch reads what an earlier one left in L2."""
    return max(lo, min(hi, -(-3 * L2_BYTES // max(1, bytes_per_set))))


def device_activations(m: int, k: int, p: float, sigma: float, gen, dev):
    """Seeded synthetic activations drawn on the device, for timing only: bf16
    N(0,1) with a fraction p of entries replaced by N(0, sigma) outliers."""
    import torch
    x = torch.randn((m, k), generator=gen, device=dev, dtype=torch.float32)
    mask = torch.rand((m, k), generator=gen, device=dev) < p
    x = torch.where(mask, torch.randn((m, k), generator=gen, device=dev) * sigma, x)
    return x.to(torch.bfloat16)


def kernel_timings(wl: dict, dev, sms: int, hbm: float, fp8_peak: float, steps: int, warmup: int,
                   decode_variants: bool = True) -> dict:
    """Isolated device timings of one workload's kernels, each in its own loop
    over rotating inputs larger than L2: the GEMM, the activation quantizer
    (with both scale layouts, as fp8q_quant_act emits them) and the fused
    linear. Each loop is timed twice, launched back to back on the stream and
    captured in a CUDA graph; fractions use the graph figure (no host launch
    work between kernels), the stream figure is reported beside it."""
    import torch
    from fp8_block_scaled_group_b200 import api
    m, n, k = wl["m"], wl["n"], wl["k"]
    g, mp = k // 128, api.m_pad(m)
    gen = torch.Generator(device=dev)
    gen.manual_seed(7000 + wl["number"] * 131 + m)
    reps = max(steps, 20)

    def both(fn, nsets):
        for i in range(max(warmup, nsets)):
            fn(i)
        torch.cuda.synchronize()
        st = stream_loop_ms(fn, max(reps, 2 * nsets))
        gr = graph_loop_ms(fn, max(reps, 2 * nsets))
        return st * 1e3, gr * 1e3

    out = {"m": m, "n": n, "k": k}
    # activation quantizer
    qb = quant_bytes(m, k)
    nq = rotation(qb)
    xs = [device_activations(m, k, wl["p"], wl["sigma"], gen, dev) for _ in range(min(nq, 3))]
    xs += [xs[i % len(xs)].clone() for i in range(len(xs), nq)]
    qo = [(torch.empty((m, k), dtype=torch.uint8, device=dev), torch.empty((m, g), dtype=torch.float32, device=dev),
           torch.empty((g, mp), dtype=torch.float32, device=dev)) for _ in range(nq)]
    pick = api.quant_pick(m, k, sms)
    picked = "multi" if pick.variant == api.MULTI else "single"
    variants = ["single", "multi"] if (decode_variants and m <= 64) else [picked]
    aq = {"bound": "hbm", "bytes": qb, "picked": picked, "peak": hbm, "unit": "GB/s"}
    for name in variants:
        var = api.MULTI if name == "multi" else api.SINGLE
        st, gr = both(lambda i, var=var: api.quant_act(xs[i % nq], variant=var, out=qo[i % nq]), nq)
        aq[name] = {"us_graph": gr, "us_stream": st}
    aq["us"] = aq[picked]["us_graph"]
    aq["us_stream"] = aq[picked]["us_stream"]
    aq["achieved"] = qb / (aq["us"] * 1e-6) / 1e9
    aq["frac"] = aq["achieved"] / hbm
    aq["frac_stream"] = qb / (aq["us_stream"] * 1e-6) / 1e9 / hbm
    out["act_quant"] = aq
    del xs, qo
    torch.cuda.empty_cache()
    # GEMM and fused linear over rotating weights
    gb = gemm_hbm_bytes(m, n, k)
    ns = rotation(n * k + m * k * 3 + 2 * m * n)
    x0 = device_activations(m, k, wl["p"], wl["sigma"], gen, dev)
    q0, _, s0 = api.quant_act(x0)
    sets = []
    for i in range(ns):
        w = (torch.randn((n, k), generator=gen, device=dev, dtype=torch.float32) * 0.02).to(torch.bfloat16)
        wq, ws = api.quant_weight(w)
        del w
        sets.append(dict(x=x0 if i == 0 else x0.clone(), q=q0 if i == 0 else q0.clone(),
                         s=s0 if i == 0 else s0.clone(), wq=wq, ws=ws,
                         work=torch.empty(api.linear_workspace_bytes(m, k), dtype=torch.uint8, device=dev),
                         y=torch.empty((m, n), dtype=torch.bfloat16, device=dev)))
    st, gr = both(lambda i: api.gemm_blockscaled(sets[i % ns]["q"], sets[i % ns]["s"], sets[i % ns]["wq"],
                                                 sets[i % ns]["ws"], out=sets[i % ns]["y"]), ns)
    flops = 2.0 * m * n * k
    if m <= 64:
        gm = {"bound": "hbm", "kernel": "gemm_decode_kernel", "unit": "GB/s", "peak": hbm,
              "achieved": gb / (gr * 1e-6) / 1e9, "frac_stream": gb / (st * 1e-6) / 1e9 / hbm}
    else:
        gm = {"bound": "tensor", "kernel": "gemm_blockscaled_kernel", "unit": "TFLOP/s", "peak": fp8_peak,
              "achieved": flops / (gr * 1e-6) / 1e12, "frac_stream": flops / (st * 1e-6) / 1e12 / fp8_peak}
    gm["frac"] = gm["achieved"] / gm["peak"]
    gm.update(us_graph=gr, us_stream=st, algorithmic_bytes=gb, tflops=flops / (gr * 1e-6) / 1e12)
    out["gemm"] = gm
    st, gr = both(lambda i: api.linear(sets[i % ns]["x"], sets[i % ns]["wq"], sets[i % ns]["ws"],
                                       workspace=sets[i % ns]["work"], out=sets[i % ns]["y"]), ns)
    out["linear"] = {"us_graph": gr, "us_stream": st, "tflops_graph": flops / (gr * 1e-6) / 1e12}
    if m <= 32:
        # The one-launch decode path (the GEMM quantizes x itself) beside it.
        st, gr = both(lambda i: api.linear_decode_fused(sets[i % ns]["x"], sets[i % ns]["wq"], sets[i % ns]["ws"],
                                                        workspace=sets[i % ns]["work"], out=sets[i % ns]["y"]), ns)
        out["linear_decode_fused"] = {"us_graph": gr, "us_stream": st}
    out["rotation"] = {"quantizer_sets": nq, "gemm_sets": ns}
    del sets
    torch.cuda.empty_cache()
    return out


def decode_quant_arms(dev, sms: int, warmup: int) -> list:
    """Both activation-quantizer variants at every decode-width arm of the
    pages' table (M in 16, 17, 25 and K in 5120, 6144, 17408), each in a CUDA
    graph over rotating inputs: the picked variant must not be the slower."""
    import torch
    from fp8_block_scaled_group_b200 import api
    rows = []
    gen = torch.Generator(device=dev)
    gen.manual_seed(7777)
    for k in (5120, 6144, 17408):
        for m in (16, 17, 25):
            g, mp = k // 128, api.m_pad(m)
            nq = 16
            xs = [device_activations(m, k, 0.01, 20.0, gen, dev) for _ in range(nq)]
            qo = [(torch.empty((m, k), dtype=torch.uint8, device=dev), torch.empty((m, g), dtype=torch.float32, device=dev),
                   torch.empty((g, mp), dtype=torch.float32, device=dev)) for _ in range(nq)]
            row = {"m": m, "k": k}
            for name, var in (("single", api.SINGLE), ("multi", api.MULTI)):
                fn = lambda i, var=var: api.quant_act(xs[i % nq], variant=var, out=qo[i % nq])
                for i in range(max(warmup, nq)):
                    fn(i)
                torch.cuda.synchronize()
                row[name + "_us"] = graph_loop_ms(fn, 64) * 1e3
            row["picked"] = "multi" if api.quant_pick(m, k, sms).variant == api.MULTI else "single"
            row["faster"] = "multi" if row["multi_us"] < row["single_us"] else "single"
            rows.append(row)
    return rows


def nvfp4_hbm_bytes(m: int, n: int, k: int) -> int:
    """Algorithmic bytes of one NVFP4 GEMM: both packed operands (half a byte
    an element), their MMA-layout scales (one byte per 16 elements, rows
    padded to 128) and the bf16 output."""
    pad = lambda r: -(-r // 128) * 128
    return m * k // 2 + n * k // 2 + (pad(m) + pad(n)) * k // 16 + 2 * m * n


def nvfp4_pack_bytes(m: int, k: int) -> int:
    """Algorithmic bytes of packing an [m, k] activation for the GEMM: read
    bf16, write the packed E2M1 pairs and the MMA-layout scales."""
    return 2 * m * k + m * k // 2 + (-(-m // 128) * 128) * k // 16


def nvfp4_timings(m: int, n: int, k: int, dev, hbm: float, fp4_peak: float, steps: int, warmup: int) -> dict:
    """The NVFP4 projection arm at one shape: the packer, the block-scaled FP4
    GEMM and the fused projection (packer + GEMM), each in its own loop over
    rotating inputs larger than L2, timed in CUDA graphs and on the stream.
    The weight is a synthetic bf16 N(0, 0.02) packed with its global scale."""
    import torch
    from fp8_block_scaled_group_b200 import api
    gen = torch.Generator(device=dev)
    gen.manual_seed(9000 + m + k)
    reps = max(steps, 20)

    def both(fn, nsets):
        for i in range(max(warmup, nsets)):
            fn(i)
        torch.cuda.synchronize()
        return stream_loop_ms(fn, max(reps, 2 * nsets)) * 1e3, graph_loop_ms(fn, max(reps, 2 * nsets)) * 1e3

    gb = nvfp4_hbm_bytes(m, n, k)
    ns = rotation(gb + 2 * m * k)
    x0 = device_activations(m, k, 0.01, 20.0, gen, dev)
    sets = []
    for _ in range(ns):
        w = (torch.randn((n, k), generator=gen, device=dev, dtype=torch.float32) * 0.02).to(torch.bfloat16)
        s2w = float(w.float().abs().max().item()) / (6.0 * 448.0)
        qw, _, sfw = api.nvfp4_quant(w, s2w, row_major=False)
        del w
        qa, _, sfa = api.nvfp4_quant(x0, 1.0, row_major=False)
        sets.append(dict(x=x0.clone(), qa=qa, sfa=sfa, qw=qw, sfw=sfw, s2w=s2w,
                         work=torch.empty(api.nvfp4_linear_workspace_bytes(m, k), dtype=torch.uint8, device=dev),
                         y=torch.empty((m, n), dtype=torch.bfloat16, device=dev)))
    out = {"m": m, "n": n, "k": k}
    st, gr = both(lambda i: api.nvfp4_gemm(sets[i % ns]["qa"], sets[i % ns]["sfa"], 1.0, sets[i % ns]["qw"],
                                           sets[i % ns]["sfw"], sets[i % ns]["s2w"], out=sets[i % ns]["y"]), ns)
    flops = 2.0 * m * n * k
    if m <= 64:
        gm = {"bound": "hbm", "unit": "GB/s", "peak": hbm, "achieved": gb / (gr * 1e-6) / 1e9}
    else:
        gm = {"bound": "tensor", "unit": "TFLOP/s", "peak": fp4_peak, "achieved": flops / (gr * 1e-6) / 1e12,
              "peak_source": "measured bf16 burst x 4 (fp4:bf16 nominal ratio; an assumption, FP4 is not measured)"}
    gm.update(kernel="nvfp4_gemm_kernel", frac=gm["achieved"] / gm["peak"], us_graph=gr, us_stream=st,
              algorithmic_bytes=gb, tflops=flops / (gr * 1e-6) / 1e12)
    out["gemm"] = gm
    pb = nvfp4_pack_bytes(m, k)
    nq = rotation(pb)
    xs = [x0.clone() for _ in range(nq)]
    po = [(torch.empty((m, k // 2), dtype=torch.uint8, device=dev),
           torch.empty((api.nvfp4_sf_mma_bytes(m, k),), dtype=torch.uint8, device=dev)) for _ in range(nq)]
    import ctypes
    from fp8_block_scaled_group_b200 import _lib
    lib = _lib.load()

    def pack(i):
        q, sf = po[i % nq]
        lib.fp8q_nvfp4_quant(ctypes.c_void_p(xs[i % nq].data_ptr()), ctypes.c_void_p(q.data_ptr()), None,
                             ctypes.c_void_p(sf.data_ptr()), 1.0, m, k,
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))

    st, gr = both(pack, nq)
    out["pack"] = {"bound": "hbm", "kernel": "nvfp4_quant_kernel", "bytes": pb, "us_graph": gr, "us_stream": st,
                   "achieved": pb / (gr * 1e-6) / 1e9, "peak": hbm, "unit": "GB/s",
                   "frac": pb / (gr * 1e-6) / 1e9 / hbm}
    st, gr = both(lambda i: api.nvfp4_linear(sets[i % ns]["x"], sets[i % ns]["qw"], sets[i % ns]["sfw"],
                                             sets[i % ns]["s2w"], workspace=sets[i % ns]["work"],
                                             out=sets[i % ns]["y"]), ns)
    out["linear"] = {"us_graph": gr, "us_stream": st, "tflops_graph": flops / (gr * 1e-6) / 1e12}
    del sets, xs, po
    torch.cuda.empty_cache()
    return out


def quant_variant_sweep(dev, sms: int) -> list:
    """Both activation-quantizer variants, forced, over M x K (CUDA graphs
    of back-to-back launches over rotating inputs larger than 3x L2): the
    measurements the SINGLE/MULTI floor is derived from."""
    import torch
    from fp8_block_scaled_group_b200 import api
    rows = []
    gen = torch.Generator(device=dev)
    gen.manual_seed(4242)
    for k in (5120, 6144, 17408):
        for m in (1, 4, 8, 16, 17, 20, 24, 25, 32, 40, 48, 56, 64, 80, 96, 128, 256, 512, 1168, 4576):
            g, mp = k // 128, api.m_pad(m)
            nq = rotation(quant_bytes(m, k), hi=64)
            base = [device_activations(m, k, 0.01, 20.0, gen, dev) for _ in range(min(nq, 2))]
            xs = [base[i % len(base)] if i < len(base) else base[i % len(base)].clone() for i in range(nq)]
            qo = [(torch.empty((m, k), dtype=torch.uint8, device=dev), torch.empty((m, g), dtype=torch.float32, device=dev),
                   torch.empty((g, mp), dtype=torch.float32, device=dev)) for _ in range(nq)]
            row = {"m": m, "k": k}
            for name, var in (("single", api.SINGLE), ("multi", api.MULTI)):
                fn = lambda i, var=var: api.quant_act(xs[i % nq], variant=var, out=qo[i % nq])
                for i in range(nq):
                    fn(i)
                torch.cuda.synchronize()
                row[name + "_us"] = graph_loop_ms(fn, max(64, 2 * nq)) * 1e3
            pick = api.quant_pick(m, k, sms)
            row["multi_ctas"] = pick.multi_ctas
            row["picked"] = "multi" if pick.variant == api.MULTI else "single"
            row["faster"] = "multi" if row["multi_us"] < row["single_us"] else "single"
            rows.append(row)
            print(json.dumps(row), flush=True)
            del xs, qo, base
            torch.cuda.empty_cache()
    return rows


# The configurations besides the headline one, timed kernel by kernel:
# decode widths at both K and the M=4576 prefill at both K.
PER_CONFIG = ["decode_m25_n6144_k5120", "decode_m25_n5120_k17408",
              "prefill_m4576_n6144_k6144", "prefill_m4576_n6144_k17408"]


# ------------------------------------------------------------ CPU oracle --

def grow_sample(run, m: int, threads: int, target_s: float):
    """Rows of a step to time so that `run(rows)` takes about target_s
    seconds (or all m rows, if they take less). A small first sample carries
    fixed overheads that make it look slow, so the estimate is refined up to
    three times. Returns (rows, seconds of the last run)."""
    threads = max(threads, 1)
    rows = max(1, min(m, threads))
    t = run(rows)
    for _ in range(3):
        if t >= 0.8 * target_s or rows >= m:
            break
        grown = int(min(m, max(rows + 1, rows * target_s / max(t, 1e-3))))
        if threads <= grown < m:
            grown -= grown % threads
        rows = grown
        t = run(rows)
    return rows, t


def sample_kind(rows: int, m: int) -> str:
    """How a reference arm's ms_per_step was obtained from its timed rows."""
    if rows >= m:
        return f"measured: each step times all {m} token rows"
    return f"extrapolated: each step times {rows} of {m} token rows and scales that time to the whole step"


def cpu_oracle_sample(wl: dict, seed: int, target_s: float, threads: int, per_row: bool = False,
                      rows: int | None = None):
    """Time the oracle on a bounded sample of one step: quantize R rows of X and
    compute those R rows of the float64 reference output. Returns
    (TFLOP/s equivalent of 2*R*N*K / time, rows, seconds)."""
    import oracle
    from fp8_block_scaled_group_b200 import inputs
    m, n, k = wl["m"], wl["n"], wl["k"]
    xb = inputs.activations(m, k, seed, wl["p"], wl["sigma"])
    wb = inputs.weights(n, k, wl["number"] + 1000)
    # weight preparation is not part of the step
    wq, ws = oracle.quant_weight_rowwise(wb) if per_row else oracle.quant_weight(wb)

    def run(rows):
        t0 = time.perf_counter()
        q, s_row, _ = oracle.quant_act(np.ascontiguousarray(xb[:rows]))
        oracle.gemm_ref(q, s_row, wq, ws, threads=threads)
        return time.perf_counter() - t0

    if rows is None:
        rows, t = grow_sample(run, m, threads, target_s)
    else:
        t = run(rows)
    return 2.0 * rows * n * k / t / 1e12, rows, t


def cpu_oracle_quant(wl: dict, seed: int):
    """The oracle's activation quantizer over the step's whole [M, K]
    activation, single-threaded: (GB/s with the GPU kernel's byte count,
    seconds)."""
    import oracle
    from fp8_block_scaled_group_b200 import inputs
    m, k = wl["m"], wl["k"]
    xb = inputs.activations(m, k, seed, wl["p"], wl["sigma"])
    t0 = time.perf_counter()
    oracle.quant_act(xb)
    t = time.perf_counter() - t0
    return quant_bytes(m, k) / t / 1e9, t


def reference_arm(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload]
    threads = os.cpu_count() or 1
    per_step = max(2.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
    vals = []
    rows = None  # sized in the first warm-up step, then the same sample every step
    for i in range(args.warmup + args.steps):
        v, rows, _ = cpu_oracle_sample(wl, 1000 + wl["number"], per_step, threads, rows=rows)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    flops = 2.0 * wl["m"] * wl["n"] * wl["k"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": flops / (value * 1e12) * 1e3,
        "ms_per_step_kind": sample_kind(rows, wl["m"]),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "m": wl["m"], "n": wl["n"], "k": wl["k"]},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{rows} of {wl['m']} token rows per step (quantize + float64 GEMM rows), "
                                   f"scaled to the metric's unit"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------- our arm --

def ours_arm(args):
    import torch
    from fp8_block_scaled_group_b200 import api, inputs

    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = WORKLOADS[args.workload]
    m, n, k = wl["m"], wl["n"], wl["k"]
    g = k // 128
    seed_base = 1000 + wl["number"]

    # Input sets: each rank draws its own tokens (weak scaling).
    sets = []
    for i in range(N_SETS):
        xb = inputs.activations(m, k, rank_input_seed(seed_base, rank, i), wl["p"], wl["sigma"])
        wb = inputs.weights(n, k, seed_base + i)
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
        w = torch.from_numpy(wb.view(np.int16)).view(torch.bfloat16).to(dev)
        wq, ws = api.quant_weight_rowwise(w) if args.weight_format == "per_row" else api.quant_weight(w)
        del w
        work = torch.empty(api.linear_workspace_bytes(m, k), dtype=torch.uint8, device=dev)
        y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        sets.append(dict(x=x, wq=wq, ws=ws, work=work, y=y, xb=xb))
    # More sets (copies in distinct memory) until a pass over them moves more
    # than 3x L2, so that no step reads what an earlier step left in L2.
    n_sets = rotation(m * k * 3 + n * k + 2 * m * n, lo=N_SETS)
    for i in range(N_SETS, n_sets):
        b = sets[i % N_SETS]
        sets.append(dict(x=b["x"].clone(), wq=b["wq"].clone(), ws=b["ws"].clone(), work=torch.empty_like(b["work"]),
                         y=torch.empty_like(b["y"]), xb=b["xb"]))
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    linear_call = api.linear_decode_fused if args.decode_path == "fused" else api.linear
    if args.decode_path == "fused" and m > 32:
        raise SystemExit("--decode-path fused serves at most 32 tokens")

    def step(i):
        s = sets[i % n_sets]
        linear_call(s["x"], s["wq"], s["ws"], workspace=s["work"], out=s["y"])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    launches0 = api.launch_count()
    barrier(world)
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    hold_stream(args.steps)
    ev0.record(stream)
    for i in range(args.steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    launches = api.launch_count() - launches0
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), world)

    # Per-kernel timing, each kernel alone in its own loop over rotating
    # inputs larger than L2 (kernel_timings): the headline workload, then the
    # other configurations, and the decode-width arms of the quantizer's two
    # variants. The clocks keep being sampled throughout.
    hbm, bf16, bf16_sus, src = load_peaks()
    fp8_peak = bf16 * 2.0  # fp8 dense = 2x bf16 dense (nominal 4.5 / 2.25 PF)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    kt = kernel_timings(wl, dev, sms, hbm, fp8_peak, args.steps, args.warmup)
    per_config = {}
    if not args.no_per_config:
        for name in PER_CONFIG:
            if name != args.workload:
                per_config[name] = kernel_timings(WORKLOADS[name], dev, sms, hbm, fp8_peak, args.steps, args.warmup)
        per_config["act_quant_decode_arms"] = decode_quant_arms(dev, sms, args.warmup)
        fp4_peak = bf16 * 4.0  # fp4 dense = 4x bf16 dense (nominal 9 / 2.25 PF), an assumption
        per_config["nvfp4_prefill_m1168_n17408_k5120"] = nvfp4_timings(1168, 17408, 5120, dev, hbm, fp4_peak,
                                                                      args.steps, args.warmup)
        per_config["nvfp4_decode_m25_n6144_k5120"] = nvfp4_timings(25, 6144, 5120, dev, hbm, fp4_peak,
                                                                  args.steps, args.warmup)
    clk = clocks.stop()

    # End to end through the public call with host buffers: pinned X in,
    # fused linear, Y back to pinned host memory, every step, with the copies
    # of neighbouring steps overlapped (pipelined_e2e_ms).
    x_host = [torch.from_numpy(s["xb"].view(np.int16)).view(torch.bfloat16).pin_memory() for s in sets[:N_SETS]]
    y_host = [torch.empty((m, n), dtype=torch.bfloat16).pin_memory() for _ in range(E2E_DEPTH)]
    x_dev = [torch.empty((m, k), dtype=torch.bfloat16, device=dev) for _ in range(E2E_DEPTH)]
    y_dev = [torch.empty((m, n), dtype=torch.bfloat16, device=dev) for _ in range(E2E_DEPTH)]

    def e2e_compute(i, b):
        s = sets[i % n_sets]
        linear_call(x_dev[b], s["wq"], s["ws"], workspace=s["work"], out=y_dev[b])

    barrier(world)
    e2e_ms = max_over_ranks(
        pipelined_e2e_ms(lambda i, b: x_dev[b].copy_(x_host[i % N_SETS], non_blocking=True), e2e_compute,
                         lambda i, b: y_host[b].copy_(y_dev[b], non_blocking=True), args.steps, args.warmup)
        * args.steps, world)

    flops = 2.0 * m * n * k
    value = weak_scaling_value(flops, world, args.steps, ms_total) / 1e12
    e2e_value = weak_scaling_value(flops, world, args.steps, e2e_ms) / 1e12
    q_kernel = "quant_act_stream_kernel" if kt["act_quant"]["picked"] == "multi" else "quant_act_single_kernel"
    q_traffic = read_traffic(q_kernel, args.workload)
    gm = kt["gemm"]
    g_kernel = gm["kernel"]
    roofline = {"bound": gm["bound"], "kernel": g_kernel, "achieved": gm["achieved"], "peak": gm["peak"],
                "unit": gm["unit"], "frac": gm["frac"], "traffic": read_traffic(g_kernel, args.workload),
                "algorithmic_bytes": gm["algorithmic_bytes"], "us": gm["us_graph"], "us_stream_loop": gm["us_stream"],
                "frac_stream_loop": gm["frac_stream"], "tflops": gm["tflops"],
                "timing": "CUDA events around a CUDA graph of back-to-back launches over rotating inputs > L2; "
                          "us_stream_loop: the same launches enqueued on the stream"}
    if gm["bound"] == "hbm":
        roofline["peak_source"] = f"{src} copy bandwidth"
    else:
        roofline["peak_source"] = f"{src} bf16 burst x 2 (fp8:bf16 nominal ratio)"
        roofline["frac_of_nominal_fp8"] = gm["achieved"] / FP8_NOMINAL_TFLOPS
    aq = kt["act_quant"]
    act_quant = {"bound": "hbm", "kernel": q_kernel, "achieved": aq["achieved"], "peak": hbm, "unit": "GB/s",
                 "frac": aq["frac"], "us": aq["us"], "us_stream_loop": aq["us_stream"],
                 "frac_stream_loop": aq["frac_stream"], "bytes": aq["bytes"], "traffic": q_traffic,
                 "peak_source": f"{src} copy bandwidth",
                 "timing": "fp8q_quant_act with both scale layouts, CUDA graph of back-to-back launches over "
                           "rotating inputs > 3x L2"}
    if m <= 64:
        act_quant["variants"] = {v: aq[v] for v in ("single", "multi") if v in aq}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        v, rows, t = cpu_oracle_sample(wl, seed_base, args.cpu_seconds, threads,
                                       per_row=args.weight_format == "per_row")
        v1, rows1, t1 = cpu_oracle_sample(wl, seed_base, args.cpu_seconds / 2, 1,
                                          per_row=args.weight_format == "per_row")
        cpu = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{rows} of {m} token rows of one step (quantize + float64 GEMM rows), "
                         f"{t:.1f} s, scaled to TFLOP/s",
               "single_thread": {"value": v1, "unit": "TFLOP/s", "cores": 1,
                                 "sample": f"{rows1} of {m} token rows, {t1:.1f} s"}}
        qv, qt = cpu_oracle_quant(wl, seed_base)
        cpu["quantizer"] = {"value": qv, "unit": "GB/s", "cores": 1,
                            "sample": f"the whole [{m}, {k}] activation, {qt:.2f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
            "config": {"workload": args.workload, "m": m, "n": n, "k": k, "parallelism": f"replicas{world}",
                       "weight_format": args.weight_format, "decode_path": args.decode_path,
                       "l2": f"{n_sets} rotating input sets ({n_sets * (m * k * 3 + n * k + m * n * 2) / 1e6:.0f} MB) "
                             f"for the step; kernel loops rotate > 3x L2"},
            "roofline": roofline,
            "act_quant": act_quant,
            "linear_us": {"stream_loop": kt["linear"]["us_stream"], "graph": kt["linear"]["us_graph"]},
            "per_config": per_config,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": m * k * 2,
                    "d2h_bytes_per_step": m * n * 2,
                    "overlap": E2E_OVERLAP},
            "gpu_launches": int(sum_over_ranks(launches, world)),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    barrier(world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


_FFN_ORACLE_W = {}


def ffn_oracle_sample(wl: dict, threads: int, target_s: float = 10.0, rows: int | None = None):
    """Time the oracle's FFN on a bounded sample of one step's token rows;
    returns (TFLOP/s equivalent, rows, seconds). Weight preparation is not
    part of the step and is done once."""
    import oracle
    from fp8_block_scaled_group_b200 import inputs
    m, d, i = wl["m"], wl["d"], wl["i"]
    xb = inputs.activations(m, d, wl["seed"])
    key = (d, i, wl["seed"])
    if key not in _FFN_ORACLE_W:
        _FFN_ORACLE_W[key] = (*oracle.quant_weight(inputs.weights(2 * i, d, wl["seed"])),
                              *oracle.quant_weight(inputs.weights(d, i, wl["seed"] + 1)))
    wq_gu, ws_gu, wq_dn, ws_dn = _FFN_ORACLE_W[key]

    def run(rows):
        t0 = time.perf_counter()
        oracle.ffn_ref(np.ascontiguousarray(xb[:rows]), wq_gu, ws_gu, wq_dn, ws_dn, threads=threads)
        return time.perf_counter() - t0

    if rows is None:
        rows, t = grow_sample(run, m, threads, target_s)
    else:
        t = run(rows)
    flops = 2.0 * rows * d * 2 * i + 2.0 * rows * i * d
    return flops / t / 1e12, rows, t


def ffn_reference_arm(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    wl = FFN_WORKLOADS[args.workload]
    threads = os.cpu_count() or 1
    vals = []
    rows = None  # sized in the first warm-up step, then the same sample every step
    per_step = max(2.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
    for j in range(args.warmup + args.steps):
        v, rows, _ = ffn_oracle_sample(wl, threads, target_s=per_step, rows=rows)
        if j >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    m, d, i = wl["m"], wl["d"], wl["i"]
    flops = 2.0 * m * d * 2 * i + 2.0 * m * i * d
    print(json.dumps({
        "impl": "reference", "metric": FFN_METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": flops / (value * 1e12) * 1e3, "higher_is_better": True, "scaling": "weak",
        "ms_per_step_kind": sample_kind(rows, m),
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "m": m, "d": d, "i": i},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{rows} of {m} token rows per step, scaled to the metric's unit"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)
    return 0


def ffn_arm(args):
    """One step = one fp8q_ffn call: quant(x), gate|up GEMM, SiLU*up + quant, down GEMM."""
    import torch
    from fp8_block_scaled_group_b200 import api, inputs

    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = FFN_WORKLOADS[args.workload]
    m, d, i = wl["m"], wl["d"], wl["i"]
    sets = []
    for j in range(N_SETS):
        xb = inputs.activations(m, d, rank_input_seed(wl["seed"], rank, j))
        to_dev = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(dev)
        wgu, wsgu = api.quant_weight(to_dev(inputs.weights(2 * i, d, wl["seed"] + 2 * j)))
        wdn, wsdn = api.quant_weight(to_dev(inputs.weights(d, i, wl["seed"] + 2 * j + 1)))
        work = torch.empty(api.ffn_workspace_layout(m, d, i)[5], dtype=torch.uint8, device=dev)
        sets.append(dict(x=to_dev(xb), xb=xb, w=(wgu, wsgu, wdn, wsdn), work=work,
                         y=torch.empty((m, d), dtype=torch.bfloat16, device=dev)))
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def step(j):
        s = sets[j % N_SETS]
        api.ffn(s["x"], *s["w"], workspace=s["work"], out=s["y"])

    counted = {}

    def timed(fn, steps):
        for j in range(args.warmup):
            fn(j)
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(int(2e6 + 2e5 * steps))
        l0 = api.launch_count()
        e0.record(stream)
        for j in range(steps):
            fn(j)
        e1.record(stream)
        counted[fn.__name__] = api.launch_count() - l0
        torch.cuda.synchronize()
        barrier(world)
        return max_over_ranks(e0.elapsed_time(e1), world) / steps

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ms = timed(step, args.steps)
    launches = counted["step"]
    # The activation step alone, over each set's own gate|up output.
    mids = [api.ffn_intermediates(s["work"], m, d, i) for s in sets]
    act_out = [(mid["q_h"], None, mid["s_h_kmajor"]) for mid in mids]

    def act(j):
        gu = mids[j % N_SETS]["gate_up"]
        api.silu_mul_quant(gu[:, :i], gu[:, i:], out=act_out[j % N_SETS])

    act_ms = timed(act, args.steps)

    def gate_up(j):
        mid = mids[j % N_SETS]
        s = sets[j % N_SETS]
        api.gemm_blockscaled(mid["q_x"], mid["s_x_kmajor"], s["w"][0], s["w"][1], out=mid["gate_up"])

    gu_ms = timed(gate_up, args.steps)
    clk = clocks.stop()

    x_host = [torch.from_numpy(s["xb"].view(np.int16)).view(torch.bfloat16).pin_memory() for s in sets]
    y_host = [torch.empty((m, d), dtype=torch.bfloat16).pin_memory() for _ in range(E2E_DEPTH)]
    x_dev = [torch.empty((m, d), dtype=torch.bfloat16, device=dev) for _ in range(E2E_DEPTH)]
    y_dev = [torch.empty((m, d), dtype=torch.bfloat16, device=dev) for _ in range(E2E_DEPTH)]

    def e2e(j, b):
        s = sets[j % N_SETS]
        api.ffn(x_dev[b], *s["w"], workspace=s["work"], out=y_dev[b])

    barrier(world)
    e2e_ms = max_over_ranks(
        pipelined_e2e_ms(lambda j, b: x_dev[b].copy_(x_host[j % N_SETS], non_blocking=True), e2e,
                         lambda j, b: y_host[b].copy_(y_dev[b], non_blocking=True), args.steps, args.warmup),
        world)

    flops = 2.0 * m * d * 2 * i + 2.0 * m * i * d
    hbm, bf16, _, src = load_peaks()
    fp8_peak = 2.0 * bf16
    act_bytes = m * i * 4 + m * i + 4 * (i // 128) * (-(-m // 16) * 16)
    gu_flops = 2.0 * m * 2 * i * d
    if m <= 64:
        gu_bytes = gemm_hbm_bytes(m, 2 * i, d)
        roofline = {"bound": "hbm", "kernel": "gemm_decode_kernel (gate|up)", "achieved": gu_bytes / (gu_ms * 1e-3) / 1e9,
                    "peak": hbm, "unit": "GB/s", "frac": gu_bytes / (gu_ms * 1e-3) / 1e9 / hbm,
                    "traffic": read_traffic("gemm_decode_kernel", args.workload),
                    "us": gu_ms * 1e3, "peak_source": f"{src} copy bandwidth"}
    else:
        tf = gu_flops / (gu_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "kernel": "gemm_blockscaled_kernel (gate|up)", "achieved": tf,
                    "peak": fp8_peak, "unit": "TFLOP/s", "frac": tf / fp8_peak,
                    "traffic": read_traffic("gemm_blockscaled_kernel", args.workload),
                    "us": gu_ms * 1e3, "peak_source": f"{src} bf16 burst x 2 (fp8:bf16 nominal ratio)",
                    "frac_of_nominal_fp8": tf / FP8_NOMINAL_TFLOPS}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        v, rows, t = ffn_oracle_sample(wl, threads, target_s=args.cpu_seconds)
        v1, rows1, t1 = ffn_oracle_sample(wl, 1, target_s=args.cpu_seconds / 2)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{rows} of {m} token rows of one FFN step, {t:.1f} s, scaled to TFLOP/s",
               "single_thread": {"value": v1, "unit": "TFLOP/s", "cores": 1,
                                 "sample": f"{rows1} of {m} token rows, {t1:.1f} s"}}
    if rank == 0:
        line = {
            "metric": FFN_METRIC, "value": weak_scaling_value(flops, world, 1, ms) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
            "data": "synthetic",
            "config": {"workload": args.workload, "m": m, "d": d, "i": i, "parallelism": f"replicas{world}",
                       "l2": f"{N_SETS} rotating input sets (weights {N_SETS * 3 * i * d / 1e6:.0f} MB) > L2"},
            "roofline": roofline,
            "act_silu_mul_quant": {"bound": "hbm", "kernel": "silu_mul_quant_kernel",
                                   "achieved": act_bytes / (act_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                                   "frac": act_bytes / (act_ms * 1e-3) / 1e9 / hbm, "us": act_ms * 1e3,
                                   "bytes": act_bytes,
                                   "traffic": read_traffic("silu_mul_quant_kernel", args.workload)},
            "cpu_baseline": cpu,
            "e2e": {"value": weak_scaling_value(flops, world, 1, e2e_ms) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": m * d * 2, "d2h_bytes_per_step": m * d * 2,
                    "overlap": E2E_OVERLAP},
            "gpu_launches": int(sum_over_ranks(launches, world)),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    barrier(world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def nvfp4_oracle_sample(wl: dict, threads: int, target_s: float, rows: int | None = None):
    """The oracle's NVFP4 projection on a bounded sample of token rows:
    pack those rows of x, then their float64 reference rows. Weight packing
    is not part of the step and is done once. Returns (TFLOP/s, rows, s)."""
    import oracle
    from fp8_block_scaled_group_b200 import inputs
    m, n, k = wl["m"], wl["n"], wl["k"]
    xb = inputs.activations(m, k, wl["seed"])
    key = ("nvfp4", n, k, wl["seed"])
    if key not in _FFN_ORACLE_W:
        wb = inputs.weights(n, k, wl["seed"] + 1)
        s2w = oracle.nvfp4_global_scale(wb)
        _FFN_ORACLE_W[key] = (*oracle.nvfp4_quant(wb, s2w), s2w)
    qw, sfw, s2w = _FFN_ORACLE_W[key]

    def run(r):
        t0 = time.perf_counter()
        qa, sfa = oracle.nvfp4_quant(np.ascontiguousarray(xb[:r]), 1.0)
        oracle.nvfp4_gemm_ref(qa, sfa, 1.0, qw, sfw, s2w)
        return time.perf_counter() - t0

    if rows is None:
        rows, t = grow_sample(run, m, threads, target_s)
    else:
        t = run(rows)
    return 2.0 * rows * n * k / t / 1e12, rows, t


def nvfp4_reference_arm(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    wl = NVFP4_WORKLOADS[args.workload]
    threads = os.cpu_count() or 1
    per_step = max(2.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
    vals, rows = [], None
    for j in range(args.warmup + args.steps):
        v, rows, _ = nvfp4_oracle_sample(wl, threads, per_step, rows=rows)
        if j >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    m, n, k = wl["m"], wl["n"], wl["k"]
    print(json.dumps({
        "impl": "reference", "metric": NVFP4_METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 2.0 * m * n * k / (value * 1e12) * 1e3, "higher_is_better": True, "scaling": "weak",
        "ms_per_step_kind": sample_kind(rows, m),
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "m": m, "n": n, "k": k},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{rows} of {m} token rows per step, scaled to the metric's unit"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)
    return 0


def nvfp4_arm(args):
    """One step = one fp8q_nvfp4_linear call: pack x (E2M1 + E4M3 block
    scales) and the block-scaled FP4 GEMM against a packed weight."""
    import torch
    from fp8_block_scaled_group_b200 import api, inputs

    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = NVFP4_WORKLOADS[args.workload]
    m, n, k = wl["m"], wl["n"], wl["k"]
    to_dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(dev)
    sets = []
    for j in range(N_SETS):
        xb = inputs.activations(m, k, rank_input_seed(wl["seed"], rank, j))
        w = to_dev(inputs.weights(n, k, wl["seed"] + 1 + j))
        s2w = float(w.float().abs().max().item()) / (6.0 * 448.0)
        qw, _, sfw = api.nvfp4_quant(w, s2w, row_major=False)
        del w
        sets.append(dict(x=to_dev(xb), xb=xb, qw=qw, sfw=sfw, s2w=s2w,
                         work=torch.empty(api.nvfp4_linear_workspace_bytes(m, k), dtype=torch.uint8, device=dev),
                         y=torch.empty((m, n), dtype=torch.bfloat16, device=dev)))
    n_sets = rotation(n * k // 2 + 3 * m * k + 2 * m * n, lo=N_SETS)
    for j in range(N_SETS, n_sets):
        b = sets[j % N_SETS]
        sets.append(dict(b, x=b["x"].clone(), qw=b["qw"].clone(), sfw=b["sfw"].clone(),
                         work=torch.empty_like(b["work"]), y=torch.empty_like(b["y"])))
    torch.cuda.synchronize()

    def step(j):
        s = sets[j % n_sets]
        api.nvfp4_linear(s["x"], s["qw"], s["sfw"], s["s2w"], workspace=s["work"], out=s["y"])

    for j in range(args.warmup):
        step(j)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    l0 = api.launch_count()
    ms = max_over_ranks(stream_loop_ms(step, args.steps), world)
    launches = api.launch_count() - l0
    hbm, bf16, _, src = load_peaks()
    kt = nvfp4_timings(m, n, k, dev, hbm, bf16 * 4.0, args.steps, args.warmup)
    clk = clocks.stop()
    x_host = [torch.from_numpy(s["xb"].view(np.int16)).view(torch.bfloat16).pin_memory() for s in sets[:N_SETS]]
    y_host = [torch.empty((m, n), dtype=torch.bfloat16).pin_memory() for _ in range(E2E_DEPTH)]
    x_dev = [torch.empty((m, k), dtype=torch.bfloat16, device=dev) for _ in range(E2E_DEPTH)]
    y_dev = [torch.empty((m, n), dtype=torch.bfloat16, device=dev) for _ in range(E2E_DEPTH)]

    def e2e(j, b):
        s = sets[j % n_sets]
        api.nvfp4_linear(x_dev[b], s["qw"], s["sfw"], s["s2w"], workspace=s["work"], out=y_dev[b])

    barrier(world)
    e2e_ms = max_over_ranks(
        pipelined_e2e_ms(lambda j, b: x_dev[b].copy_(x_host[j % N_SETS], non_blocking=True), e2e,
                         lambda j, b: y_host[b].copy_(y_dev[b], non_blocking=True), args.steps, args.warmup),
        world)
    flops = 2.0 * m * n * k
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        v, rows, t = nvfp4_oracle_sample(wl, threads, args.cpu_seconds)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{rows} of {m} token rows of one step (pack + float64 reference rows), {t:.1f} s"}
    if rank == 0:
        gm = kt["gemm"]
        print(json.dumps({
            "metric": NVFP4_METRIC, "value": weak_scaling_value(flops, world, 1, ms) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e2m1", "data": "synthetic",
            "config": {"workload": args.workload, "m": m, "n": n, "k": k, "parallelism": f"replicas{world}",
                       "l2": f"{n_sets} rotating input sets for the step; kernel loops rotate > 3x L2"},
            "roofline": {"bound": gm["bound"], "kernel": gm["kernel"], "achieved": gm["achieved"], "peak": gm["peak"],
                         "unit": gm["unit"], "frac": gm["frac"], "traffic": None, "us": gm["us_graph"],
                         "us_stream_loop": gm["us_stream"], "algorithmic_bytes": gm["algorithmic_bytes"],
                         "peak_source": gm.get("peak_source", f"{src} copy bandwidth")},
            "pack": kt["pack"], "linear_us": kt["linear"],
            "cpu_baseline": cpu,
            "e2e": {"value": weak_scaling_value(flops, world, 1, e2e_ms) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": m * k * 2, "d2h_bytes_per_step": m * n * 2,
                    "overlap": E2E_OVERLAP},
            "gpu_launches": int(sum_over_ranks(launches, world)),
            "clocks": clk,
        }), flush=True)
    barrier(world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(FFN_WORKLOADS) + sorted(NVFP4_WORKLOADS),
                    default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the chosen workload's kernels, not the other configurations")
    ap.add_argument("--weight-format", choices=["block128", "per_row"], default="block128",
                    help="weight scales per 128x128 block (the pages' format) or one per weight row")
    ap.add_argument("--decode-path", choices=["two_launch", "fused"], default="two_launch",
                    help="decode widths (M <= 32): quantizer + GEMM, or the GEMM with the quantizer fused in")
    ap.add_argument("--quant-sweep", action="store_true",
                    help="time both quantizer variants over M x K on cuda:0 (one JSON row each) and exit")
    ap.add_argument("--kernel-digests", action="store_true",
                    help="print the source digest of each kernel (the key of profiles/traffic.txt) and exit")
    args = ap.parse_args()
    if args.kernel_digests:
        for kname in KERNEL_SOURCES:
            print(kname, kernel_digest(kname))
        return 0
    if args.quant_sweep:
        import torch
        dev = torch.device("cuda", 0)
        quant_variant_sweep(dev, torch.cuda.get_device_properties(dev).multi_processor_count)
        return 0
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    if args.workload in FFN_WORKLOADS:
        if args.impl == "reference":
            return ffn_reference_arm(args)
        return ffn_arm(args)
    if args.workload in NVFP4_WORKLOADS:
        if args.impl == "reference":
            return nvfp4_reference_arm(args)
        return nvfp4_arm(args)
    if args.impl == "reference":
        return reference_arm(args)
    return ours_arm(args)


if __name__ == "__main__":
    sys.exit(main())

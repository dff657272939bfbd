#!/usr/bin/env python
"""Time both activation-quantizer variants over M x K on the current GPU.

The variant pick (fp8q_quant_pick) runs the multi-group quantizer once its
grid reaches a CTA floor expressed per SM, the rule of the page
"spark_model/layers/ops/fp8_act_quant_floor.rs". The floor this library uses
(two thirds of a CTA per SM) comes from this sweep on a B200; run it on
another part to re-derive the crossover.

Each point: a CUDA graph of 100 launches of one forced variant, replayed 5
times, median per-launch time. Inputs rotate over enough buffers to exceed
L2 at prefill widths. Prints one JSON object per (M, K) and writes them all
to --out.

    python -m fp8_block_scaled_group_b200.tune_quant_floor --out sweep.json
"""
from __future__ import annotations

import argparse
import json
import os
import sys

if __package__ in (None, ""):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import torch

from fp8_block_scaled_group_b200 import api

MS = [1, 4, 8, 12, 16, 17, 20, 24, 25, 28, 32, 40, 48, 56, 64, 80, 96, 128, 256, 512, 1168, 4576]
KS = [5120, 6144, 17408]
REPS = 100


def time_variant(xs, out, variant):
    nbuf = len(xs)
    for i in range(5):
        api.quant_act(xs[i % nbuf], variant=variant, out=out)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        api.quant_act(xs[0], variant=variant, out=out)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(REPS):
            api.quant_act(xs[i % nbuf], variant=variant, out=out)
    graph.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(5):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3 / REPS)
    return sorted(times)[len(times) // 2]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default="quant_floor_sweep.json")
    args = ap.parse_args()
    dev = torch.device("cuda:0")
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    rows = []
    for k in KS:
        for m in MS:
            nbuf = max(1, min(32, int(400e6 // (m * k * 3))))
            xs = [torch.randn(m, k, device=dev).to(torch.bfloat16) for _ in range(nbuf)]
            g, mp = k // 128, api.m_pad(m)
            out = (torch.empty(m, k, dtype=torch.uint8, device=dev),
                   torch.empty(m, g, dtype=torch.float32, device=dev),
                   torch.empty(g, mp, dtype=torch.float32, device=dev))
            row = {"m": m, "k": k, "sms": sms}
            for name, v in (("single", api.SINGLE), ("multi", api.MULTI)):
                row[name + "_us"] = time_variant(xs, out, v)
            row["multi_ctas"] = api.quant_pick(m, k, sms, api.MULTI).grid_x
            row["faster"] = "multi" if row["multi_us"] < row["single_us"] else "single"
            row["picked"] = "multi" if api.quant_pick(m, k, sms).variant == api.MULTI else "single"
            rows.append(row)
            print(json.dumps(row), flush=True)
            del xs
    with open(args.out, "w") as f:
        json.dump(rows, f, indent=1)


if __name__ == "__main__":
    main()

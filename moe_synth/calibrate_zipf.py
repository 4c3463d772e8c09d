"""Calibrate beta of the Zipf-skewed router correction bias.

The skewed GLM-5-shaped workload asks for per-expert token counts "from near
0 to about 10x the mean".  Its bias is e_bias[pi(r)] = beta * log p_r with
p_r proportional to r^-1.1 (r = 1..M).  This script finds, by bisection, the
beta for which the busiest expert receives ``target`` times the mean count
on the seed-0 inputs, routing with the CPU oracle's router (fp64).  The
result is stored as ZIPF_BETA_GLM5 in moe_synth/configs.py.

    python -m moe_synth.calibrate_zipf [--target 10]
"""
from __future__ import annotations

import argparse
import time

import numpy as np
import torch

import moe_synth as ms
import oracle


def counts_for(cfg, logits, beta):
    cfg = dict(cfg)
    cfg["e_bias"] = ("zipf", cfg["e_bias"][1], beta)
    bias = ms.router_bias(cfg).double().numpy()
    sel, _ = oracle.selection_scores(logits, cfg["gate"], bias)
    idx = oracle.topk_select(sel, cfg["k"])
    return np.bincount(idx.reshape(-1), minlength=cfg["M"])


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="glm5_skewed_prefill_bf16")
    ap.add_argument("--target", type=float, default=10.0)
    args = ap.parse_args()
    cfg = ms.get_config(args.config)
    t0 = time.time()
    x = ms.x_tokens(cfg).double().numpy()
    w_r = ms.router_weight(cfg).double().numpy()
    logits = oracle.router_logits(x, w_r)
    print(f"inputs + logits in {time.time() - t0:.1f}s")
    mean = cfg["T"] * cfg["k"] / cfg["M"]
    lo, hi = 0.0, 1.0
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        c = counts_for(cfg, logits, mid)
        if c.max() / mean < args.target:
            lo = mid
        else:
            hi = mid
    beta = round(0.5 * (lo + hi), 4)
    c = counts_for(cfg, logits, beta)
    print(f"beta={beta} max/mean={c.max() / mean:.2f} min={c.min()} "
          f"median/mean={np.median(c) / mean:.2f} empty={(c == 0).sum()}")


if __name__ == "__main__":
    torch.set_num_threads(max(1, torch.get_num_threads()))
    main()

"""Helpers shared by the GPU parity tests: run the CUDA path, run the oracle
on the same inputs, compare with the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

import moe_synth as ms
import oracle

# Tolerances (stated in the problem statement for bf16 inputs with fp32
# accumulation against an fp64 oracle on the same values):
Y_MAX_OVER_RMS = 2e-2      # max |y - y_ref| <= 2e-2 * rms(y_ref)
Y_MEAN_REL = 5e-3          # sum |y - y_ref| / sum |y_ref| <= 5e-3
TIE_REL = 1e-5             # near-tie band of the router selection
# fp32 arithmetic of the same values: only summation order differs.
Y_F32_MEAN_REL = 1e-5
Y_F32_MAX_OVER_RMS = 1e-4
# gate weights: fp32 logits/sigmoid/renormalisation against fp64
W_ABS = 1e-4


def np64(t):
    return t.detach().to(torch.float64).cpu().numpy()


def tol_y(cfg):
    if cfg["dtype"] == "f32":
        return Y_F32_MAX_OVER_RMS, Y_F32_MEAN_REL
    return Y_MAX_OVER_RMS, Y_MEAN_REL


class HostExperts:
    """Expert weights fetched from device tensors to fp64 host arrays on demand."""

    def __init__(self, inp):
        self.inp = inp
        self.cache = {}

    def __call__(self, e):
        if e not in self.cache:
            if len(self.cache) > 4:
                self.cache.clear()
            b1 = self.inp.get("b1")
            b2 = self.inp.get("b2")
            self.cache[e] = (np64(self.inp["w1"][e]), np64(self.inp["w2"][e]),
                             None if b1 is None else np64(b1[e]), None if b2 is None else np64(b2[e]))
        return self.cache[e]


def oracle_route(cfg, inp):
    b = inp.get("e_bias")
    return oracle.route(np64(inp["x"]), np64(inp["w_r"]), None if b is None else np64(b), cfg["k"],
                        cfg["gate"], cfg["norm_topk_prob"], cfg["alpha"], cfg["eps"],
                        cfg.get("n_group", 1) or 1, cfg.get("topk_group", 1) or 1)


def _check_grouped_topk(cfg, sel, gpu_idx):
    """Group-limited top-k: equal to the oracle's, or explained by near-ties.

    Where the GPU differs, its choice must be the top-k (per-slot near-ties
    allowed) over a set of at most topk_group groups that holds every group
    scoring clearly above the oracle's cut, and whose other groups score
    within the near-tie band of the cut."""
    n_group, topk_group, k = cfg["n_group"], cfg["topk_group"], cfg["k"]
    T, M = sel.shape
    size = M // n_group
    masked = oracle.group_limit(sel, n_group, topk_group)
    ref = oracle.topk_select(masked, k)
    differ = np.nonzero((gpu_idx != ref).any(axis=1))[0]
    for t in differ:
        row = sel[t]
        gscore = (-np.sort(-row.reshape(n_group, size), axis=1))[:, :min(2, size)].sum(axis=1)
        cut = np.sort(gscore)[::-1][topk_group - 1]
        band = TIE_REL * np.abs(gscore).max()
        picked = set((np.asarray(gpu_idx[t]) // size).tolist())
        forced = set(np.nonzero(gscore > cut + band)[0].tolist())
        groups = forced | picked
        assert len(groups) <= topk_group, f"token {t}: GPU experts span too many groups"
        assert all(gscore[g] >= cut - band for g in picked), f"token {t}: GPU took an ineligible group"
        allowed = np.repeat(np.isin(np.arange(n_group), sorted(groups)), size)
        ok, _, _ = oracle.adopt_topk(gpu_idx[t:t + 1], np.where(allowed, row, -np.inf)[None, :], TIE_REL)
        assert ok, f"token {t}: top-k inside the eligible groups differs beyond the near-tie band"
    return len(differ)


def check_routing(cfg, r, gpu_idx, gpu_w):
    """Top-k bit-exact up to near-ties (adopted), weights within W_ABS*alpha."""
    if (cfg.get("n_group", 1) or 1) > 1:
        ndiff = _check_grouped_topk(cfg, r["sel"], np.asarray(gpu_idx, dtype=np.int64))
    else:
        ok, ndiff, bad = oracle.adopt_topk(gpu_idx, r["sel"], TIE_REL)
        assert ok, f"top-k differs beyond the near-tie band at token {bad}"
    w_ref = oracle.topk_weights(gpu_idx, r["logits"], r["g"], cfg["gate"], cfg["norm_topk_prob"],
                                cfg["alpha"], cfg["eps"])
    if cfg["norm_topk_prob"] and gpu_w.size:
        # the renormalised weights of a token sum to alpha * S / (S + eps) (sigmoid; the GLM-4.5
        # note's g-bar) or to alpha (softmax over the selected experts), in fp32 to ~1e-6
        target = w_ref.sum(axis=1)
        err_sum = np.abs(np.asarray(gpu_w, np.float64).sum(axis=1) - target).max()
        assert err_sum <= 1e-6 * max(1.0, cfg["alpha"]) * cfg["k"], f"weight sum off by {err_sum}"
    err = np.abs(gpu_w - w_ref).max() if gpu_w.size else 0.0
    assert err <= W_ABS * max(1.0, cfg["alpha"]), f"gate weights off by {err}"
    return w_ref, ndiff


def check_permutation(cfg, gpu_idx, gpu_w, perm_gpu):
    """counts, offsets, slot_of, row_token bit-exact; row_w a bit-exact copy."""
    p = oracle.permute(gpu_idx, gpu_w.astype(np.float64), cfg["M"])
    assert np.array_equal(perm_gpu["counts"], p["counts"])
    assert np.array_equal(perm_gpu["offsets"], p["offsets"])
    assert np.array_equal(perm_gpu["slot_of"], p["slot_of"])
    assert np.array_equal(perm_gpu["row_token"], p["row_token"])
    assert np.array_equal(perm_gpu["row_w"].astype(np.float64), p["row_w"])
    return p


def oracle_y(cfg, inp, tokens, idx, w_ref):
    x = np64(inp["x"][torch.as_tensor(tokens, device=inp["x"].device)])
    shared = None
    if cfg.get("I_sh"):
        shared = (np64(inp["sh_w1"]), np64(inp["sh_w2"]))
    return oracle.moe_tokens(x, idx[tokens], w_ref[tokens], cfg["act"], HostExperts(inp), shared)


# Bound for inputs outside the five named workloads (edge cases whose
# outputs can have heavier tails): bf16 storage of y alone costs up to half
# an ulp, i.e. 2^-8 |y_ref|, at every element; the max criterion is applied
# to what remains.
BF16_HALF_ULP_REL = 2.0 ** -8


def check_y(cfg, y_gpu_rows, y_ref):
    m = oracle.error_metrics(y_gpu_rows, y_ref)
    max_tol, mean_tol = tol_y(cfg)
    assert m["mean_rel"] <= mean_tol, m
    if cfg.get("named") or cfg["dtype"] == "f32":
        assert m["max_over_rms"] <= max_tol, m
    else:
        y = np.asarray(y_gpu_rows, np.float64)
        rms = float(np.sqrt(np.mean(y_ref ** 2)))
        excess = np.abs(y - y_ref) - BF16_HALF_ULP_REL * np.abs(y_ref)
        m["max_excess_over_rms"] = float(excess.max() / rms)
        assert m["max_excess_over_rms"] <= max_tol, m
    return m


def sample_tokens(cfg, counts, row_token, offsets, n_random=6, seed=0):
    """A deterministic handful of tokens: both ends, random ones, the last row
    of the busiest expert's segment and the token of the smallest segment."""
    T = cfg["T"]
    rng = np.random.default_rng(seed)
    toks = {0, 1, T // 2, T - 2, T - 1}
    toks.update(rng.integers(0, T, n_random).tolist())
    busiest = int(np.argmax(counts))
    toks.add(int(row_token[offsets[busiest + 1] - 1]))
    nz = np.nonzero(counts)[0]
    smallest = int(nz[np.argmin(counts[nz])])
    toks.add(int(row_token[offsets[smallest]]))
    return np.array(sorted(t for t in toks if 0 <= t < T), dtype=np.int64)


def swap_token_tiles(cnt, max_width=256):
    """Token tiles of one expert segment of ``cnt`` rows as the library's
    tokens-on-N expert GEMM cuts it: the fewest tiles of at most 256 rows,
    all of one width rounded up to a multiple of 16, the last one ragged.
    Returns (first row, rows) of each tile, relative to the segment."""
    if cnt <= 0:
        return []
    n0 = -(-cnt // max_width)
    width = (-(-cnt // n0) + 15) // 16 * 16
    return [(r0, min(width, cnt - r0)) for r0 in range(0, cnt, width)]


def tile_tokens(cfg, counts, row_token, offsets, seed=0):
    """Tokens whose outputs together exercise every token tile of the
    full-size expert GEMMs: for each expert segment and each of its token
    tiles, the tokens of the tile's first row, last row and one row between;
    for the shared expert (one segment of all T tokens) the first and last
    token of each 256-token tile; plus the extremes of sample_tokens."""
    rng = np.random.default_rng(seed)
    toks = set(sample_tokens(cfg, counts, row_token, offsets).tolist())
    for e in range(len(counts)):
        base = int(offsets[e])
        for r0, n in swap_token_tiles(int(counts[e])):
            for r in {r0, r0 + n - 1, r0 + int(rng.integers(0, n))}:
                toks.add(int(row_token[base + r]))
    if cfg.get("I_sh"):
        for r0, n in swap_token_tiles(cfg["T"]):
            toks.update((r0, r0 + n - 1))
    return np.array(sorted(toks), dtype=np.int64)


def gpu_inputs(cfg):
    return ms.layer_inputs(cfg, "cuda")

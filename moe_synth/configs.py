"""Workload definitions for the sparse MoE FFN layer forward.

Each entry gives the layer's shapes, router and expert kind, and the value
distributions of its synthetic inputs.  Field meanings:

  dtype          "f32" or "bf16": type of x, W_r, the expert weights, biases, y
  T, D, M, k     tokens, model width, routed experts, experts per token
  gate           "softmax" (GLaM note, eq. r_t and S_t) or "sigmoid_bias"
                 (GLM-4.5 shared-expert note, "How it works")
  act            "gelu_tanh": E(x) = W2 GELU_tanh(W1 x + b1) + b2 (GLaM note,
                 eq. FFN); "swiglu": E(x) = W_down(SiLU(W_gate x) * W_up x)
  I              expert hidden width (H of the GELU FFN, d_moe of SwiGLU)
  has_bias       GELU experts carry b1, b2
  norm_topk_prob renormalise the k selected gate values
  alpha          routed_scaling_factor
  eps            added to the renormalisation denominator (sigmoid router)
  I_sh           width of the always-on shared SwiGLU expert (0 = none)
  w_r_std        standard deviation of W_r
  bias_std       standard deviation of b1, b2
  e_bias         None, ("uniform", lo, hi), ("zipf", s, beta) or ("const", v)

Expert weights are N(0, 1/fan_in) (variance 1/fan_in); x is N(0, 1).
"""
from __future__ import annotations

import math

# beta of the Zipf-skewed correction bias: calibrated by
# moe_synth/calibrate_zipf.py on the seed-0 inputs so that the busiest
# expert receives about 10x the mean number of tokens.
ZIPF_BETA_GLM5 = 0.0555

CONFIGS = {
    # Tiny GLaM-style layer, fp32 (correctness only)
    "glam_tiny_f32": dict(
        dtype="f32", T=256, D=64, M=8, k=2, gate="softmax", act="gelu_tanh",
        I=256, has_bias=1, norm_topk_prob=1, alpha=1.0, eps=1e-20, I_sh=0,
        w_r_std=0.02, bias_std=0.01, e_bias=None),
    # GLaM-style prefill layer, bf16
    "glam_prefill_bf16": dict(
        dtype="bf16", T=8192, D=2048, M=64, k=2, gate="softmax", act="gelu_tanh",
        I=8192, has_bias=1, norm_topk_prob=1, alpha=1.0, eps=1e-20, I_sh=0,
        w_r_std=1.0 / math.sqrt(2048), bias_std=0.01, e_bias=None),
    # GLM-4.5-shaped decode layer, bf16 (memory-bound)
    "glm45_decode_bf16": dict(
        dtype="bf16", T=32, D=5120, M=160, k=8, gate="sigmoid_bias", act="swiglu",
        I=1536, has_bias=0, norm_topk_prob=1, alpha=2.5, eps=1e-20, I_sh=1536,
        w_r_std=1.0 / math.sqrt(5120), bias_std=0.0, e_bias=("uniform", -0.1, 0.1)),
    # GLM-4.5-shaped prefill layer, bf16
    "glm45_prefill_bf16": dict(
        dtype="bf16", T=16384, D=5120, M=160, k=8, gate="sigmoid_bias", act="swiglu",
        I=1536, has_bias=0, norm_topk_prob=1, alpha=2.5, eps=1e-20, I_sh=1536,
        w_r_std=0.02, bias_std=0.0, e_bias=("uniform", -0.1, 0.1)),
    # GLM-5-shaped prefill layer with Zipf-skewed expert load, bf16
    "glm5_skewed_prefill_bf16": dict(
        dtype="bf16", T=16384, D=6144, M=256, k=8, gate="sigmoid_bias", act="swiglu",
        I=2048, has_bias=0, norm_topk_prob=1, alpha=1.0, eps=1e-20, I_sh=2048,
        w_r_std=0.02, bias_std=0.0, e_bias=("zipf", 1.1, ZIPF_BETA_GLM5)),
}

# Small cases: several tiles and ragged tails, quick for the oracle.
TEST_CONFIGS = {
    "glam_small_bf16": dict(
        dtype="bf16", T=333, D=192, M=8, k=2, gate="softmax", act="gelu_tanh",
        I=320, has_bias=1, norm_topk_prob=1, alpha=1.0, eps=1e-20, I_sh=0,
        w_r_std=0.05, bias_std=0.01, e_bias=None),
    "glm_small_bf16": dict(
        dtype="bf16", T=300, D=256, M=16, k=4, gate="sigmoid_bias", act="swiglu",
        I=192, has_bias=0, norm_topk_prob=1, alpha=2.5, eps=1e-20, I_sh=128,
        w_r_std=0.05, bias_std=0.0, e_bias=("uniform", -0.1, 0.1)),
    "glm_medium_bf16": dict(
        dtype="bf16", T=1000, D=512, M=32, k=8, gate="sigmoid_bias", act="swiglu",
        I=256, has_bias=0, norm_topk_prob=1, alpha=1.0, eps=1e-20, I_sh=320,
        w_r_std=0.05, bias_std=0.0, e_bias=("zipf", 1.1, 0.2)),
    "glm_small_f32": dict(
        dtype="f32", T=77, D=64, M=12, k=3, gate="sigmoid_bias", act="swiglu",
        I=96, has_bias=0, norm_topk_prob=1, alpha=2.5, eps=1e-20, I_sh=64,
        w_r_std=0.05, bias_std=0.0, e_bias=("uniform", -0.1, 0.1)),
    "glm_grouped_bf16": dict(
        dtype="bf16", T=700, D=256, M=64, k=6, gate="sigmoid_bias", act="swiglu",
        I=128, has_bias=0, norm_topk_prob=1, alpha=2.5, eps=1e-20, I_sh=128,
        w_r_std=0.05, bias_std=0.0, e_bias=("uniform", -0.1, 0.1), n_group=8, topk_group=3),
    "glm_grouped_f32": dict(
        dtype="f32", T=90, D=64, M=32, k=4, gate="sigmoid_bias", act="swiglu",
        I=64, has_bias=0, norm_topk_prob=1, alpha=1.0, eps=1e-20, I_sh=0,
        w_r_std=0.05, bias_std=0.0, e_bias=("uniform", -0.1, 0.1), n_group=4, topk_group=2),
    "glam_nonorm_f32": dict(
        dtype="f32", T=50, D=64, M=8, k=2, gate="softmax", act="gelu_tanh",
        I=128, has_bias=1, norm_topk_prob=0, alpha=1.0, eps=1e-20, I_sh=0,
        w_r_std=0.05, bias_std=0.01, e_bias=None),
}


# Dense FFN layers (no router): the "GLaM" note's DenseFFN between its MoE
# layers (the GLaM prefill layer's own shapes), and small test cases.
DENSE_CONFIGS = {
    "glam_dense_bf16": dict(
        dtype="bf16", T=8192, D=2048, I=8192, act="gelu_tanh", has_bias=1, bias_std=0.01),
    "glam_dense_small_bf16": dict(
        dtype="bf16", T=333, D=192, I=320, act="gelu_tanh", has_bias=1, bias_std=0.01),
    "glm_dense_small_bf16": dict(
        dtype="bf16", T=300, D=256, I=384, act="swiglu", has_bias=0, bias_std=0.0),
    "glm_dense_small_f32": dict(
        dtype="f32", T=77, D=64, I=96, act="swiglu", has_bias=0, bias_std=0.0),
    "glam_dense_small_f32": dict(
        dtype="f32", T=50, D=64, I=128, act="gelu_tanh", has_bias=1, bias_std=0.01),
}


def get_config(name: str, **overrides) -> dict:
    base = CONFIGS.get(name) or TEST_CONFIGS.get(name) or DENSE_CONFIGS.get(name)
    if base is None:
        raise KeyError(name)
    cfg = dict(base)
    cfg["name"] = name
    cfg.setdefault("seed", 0)
    cfg.update(overrides)
    # one of the five named workloads, unchanged
    cfg["named"] = name in CONFIGS and not overrides
    return cfg


def all_config_names():
    """Names of the MoE layer workloads (named and test cases)."""
    return list(CONFIGS) + list(TEST_CONFIGS)


def dense_config_names():
    return list(DENSE_CONFIGS)

"""The CPU backward oracle against its pins (finite differences of the pinned
forward, invariants), and planted mistakes in a patched copy of it, each of
which some pin must catch."""
import importlib.util
import os

import numpy as np
import pytest

import oracle.moe_backward
from oracle_pins_backward import BWD_PINS

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "moe_backward.py")


@pytest.mark.parametrize("pin", BWD_PINS, ids=lambda f: f.__name__)
def test_backward_pin(pin):
    pin(oracle.moe_backward)


def fresh():
    spec = importlib.util.spec_from_file_location("oracle._backward_mutant", SRC)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def caught(mod):
    for pin in BWD_PINS:
        try:
            pin(mod)
        except AssertionError:
            return pin.__name__
    return None


def m_silu_grad_no_product_term(B):
    B.silu_grad = lambda v: B.F.sigmoid(v)


def m_gelu_grad_no_cubic(B):
    c = np.sqrt(2.0 / np.pi)

    def g(v):
        v = np.asarray(v, np.float64)
        th = np.tanh(c * (v + 0.044715 * v ** 3))
        return 0.5 * (1.0 + th) + 0.5 * v * (1.0 - th * th) * c
    B.gelu_tanh_grad = g


def m_router_no_centering(B):
    orig = B.router_backward

    def rb(idx, dw, logits, g, gate, norm, alpha, eps):
        if gate != "softmax" or not norm:
            return orig(idx, dw, logits, g, gate, norm, alpha, eps)
        l = np.asarray(logits, np.float64)
        dl = np.zeros_like(l)
        for t in range(l.shape[0]):
            es = np.asarray(idx[t])
            q = np.exp(l[t, es] - l[t, es].max())
            q = q / q.sum()
            dl[t, es] = alpha * q * np.asarray(dw)[t]
        return dl
    B.router_backward = rb


def m_router_no_sigmoid_slope(B):
    orig = B.router_backward

    def rb(idx, dw, logits, g, gate, norm, alpha, eps):
        dl = orig(idx, dw, logits, g, gate, norm, alpha, eps)
        if gate == "sigmoid_bias":
            gg = np.asarray(g, np.float64)
            with np.errstate(divide="ignore", invalid="ignore"):
                dl = np.where(dl != 0, dl / (gg * (1 - gg)), 0.0)
        return dl
    B.router_backward = rb


def m_router_sigmoid_no_norm_term(B):
    orig = B.router_backward

    def rb(idx, dw, logits, g, gate, norm, alpha, eps):
        if gate == "sigmoid_bias" and norm:
            return orig(idx, dw, logits, g, gate, False, alpha, eps)
        return orig(idx, dw, logits, g, gate, norm, alpha, eps)
    B.router_backward = rb


def _patch_moe(B, **changes):
    orig_ffn = B.expert_ffn_backward
    if "scaled_dw" in changes:
        def ffn(xe, act, w1e, w2e, b1e, b2e, dout):
            r = orig_ffn(xe, act, w1e, w2e, b1e, b2e, dout)
            r = dict(r)
            r["out"] = r["out"] * 0.5        # dw from a half-scaled output
            return r
        B.expert_ffn_backward = ffn
    if "no_router_dx" in changes:
        orig_moe = B.moe_backward

        def moe(cfg, inp, dy, idx=None):
            r = orig_moe(cfg, inp, dy, idx)
            r = dict(r)
            r["dx"] = r["dx"] - r["dl"] @ np.asarray(inp["w_r"], np.float64).T
            return r
        B.moe_backward = moe


def m_dw_from_scaled_output(B):
    _patch_moe(B, scaled_dw=True)


def m_no_router_term_in_dx(B):
    _patch_moe(B, no_router_dx=True)


def m_no_shared_dx(B):
    orig = B.moe_backward

    def moe(cfg, inp, dy, idx=None):
        r = dict(orig(cfg, inp, dy, idx))
        if cfg.get("I_sh"):
            gs = B.expert_ffn_backward(inp["x"], "swiglu", inp["sh_w1"], inp["sh_w2"], None, None, dy)
            r["dx"] = r["dx"] - gs["dx"]
        return r
    B.moe_backward = moe


def m_swiglu_halves_swapped(B):
    orig = B.expert_ffn_backward

    def ffn(xe, act, w1e, w2e, b1e, b2e, dout):
        r = dict(orig(xe, act, w1e, w2e, b1e, b2e, dout))
        if act == "swiglu":
            I = r["dw1"].shape[0] // 2
            r["dw1"] = np.concatenate([r["dw1"][I:], r["dw1"][:I]])
        return r
    B.expert_ffn_backward = ffn


def m_gelu_grad_without_b1(B):
    orig = B.expert_ffn_backward

    def ffn(xe, act, w1e, w2e, b1e, b2e, dout):
        if act != "gelu_tanh" or b1e is None:
            return orig(xe, act, w1e, w2e, b1e, b2e, dout)
        r = dict(orig(xe, act, w1e, w2e, b1e, b2e, dout))
        r2 = orig(xe, act, w1e, w2e, np.zeros_like(np.asarray(b1e)), b2e, dout)
        r["dx"] = r2["dx"]
        return r
    B.expert_ffn_backward = ffn


def m_load_cv_sample_std(B):
    orig = B.expert_load

    def el(idx, M):
        s = dict(orig(idx, M))
        c = s["counts"]
        s["cv"] = float(np.std(c, ddof=1) / c.mean())
        return s
    B.expert_load = el


MUTANTS = [m_silu_grad_no_product_term, m_gelu_grad_no_cubic, m_router_no_centering,
           m_router_no_sigmoid_slope, m_router_sigmoid_no_norm_term, m_dw_from_scaled_output,
           m_no_router_term_in_dx, m_no_shared_dx, m_swiglu_halves_swapped, m_gelu_grad_without_b1,
           m_load_cv_sample_std]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda f: f.__name__)
def test_backward_mutant_is_caught(mutant):
    mod = fresh()
    mutant(mod)
    assert caught(mod) is not None, mutant.__name__

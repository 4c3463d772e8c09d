"""Checks that pin the CPU backward oracle to facts outside its own code.

Each ``pin_*`` takes the backward module and raises AssertionError when it
disagrees.  The independent side is the derivative itself: central finite
differences, in fp64, of the loss L = sum(dy * y) computed by the forward
oracle (pinned on its own by oracle_pins.py), on tiny layers of every router
and expert variant.  A perturbation that changes the discrete top-k choice is
not a derivative of the layer, so such elements are skipped (and counted).
Besides: the shift invariance of softmax weights, and the load statistic
against the standard library.
"""
from __future__ import annotations

import math
import statistics

import numpy as np

from oracle import moe_oracle as FWD
from oracle_pins import tiny_inputs

BWD_TINY = [
    # "GLaM": renormalised softmax top-2, GELU experts with biases
    dict(T=6, D=5, M=4, k=2, gate="softmax", act="gelu_tanh", I=3,
         norm_topk_prob=1, alpha=1.0, eps=1e-20, I_sh=0),
    # GLM-4.5 / GLM-5: sigmoid + correction bias, normalised, scaled, SwiGLU + shared expert
    dict(T=6, D=5, M=4, k=2, gate="sigmoid_bias", act="swiglu", I=3,
         norm_topk_prob=1, alpha=2.5, eps=1e-20, I_sh=2),
    # full-softmax weights (not renormalised) with SwiGLU and a shared expert
    dict(T=5, D=4, M=5, k=3, gate="softmax", act="swiglu", I=2,
         norm_topk_prob=0, alpha=1.5, eps=1e-20, I_sh=3),
    # sigmoid without normalisation, GELU with biases
    dict(T=5, D=4, M=4, k=2, gate="sigmoid_bias", act="gelu_tanh", I=3,
         norm_topk_prob=0, alpha=0.7, eps=1e-20, I_sh=0),
    # group-limited sigmoid router (8 experts in 4 groups, 2 kept)
    dict(T=6, D=4, M=8, k=2, gate="sigmoid_bias", act="swiglu", I=2,
         norm_topk_prob=1, alpha=2.5, eps=1e-20, I_sh=2, n_group=4, topk_group=2),
]

PARAMS = ("x", "w_r", "w1", "w2", "b1", "b2", "sh_w1", "sh_w2")
GRAD_OF = {"x": "dx", "w_r": "dw_r", "w1": "dw1", "w2": "dw2", "b1": "db1", "b2": "db2",
           "sh_w1": "dsh_w1", "sh_w2": "dsh_w2"}


def _loss(cfg, inp, dy):
    out = FWD.moe_forward(cfg, inp)
    return float(np.sum(dy * out["y"])), out["idx"]


def _fd_check(B, cfg, seed, h=1e-5):
    inp = tiny_inputs(cfg, seed)
    rng = np.random.default_rng(seed + 1000)
    dy = rng.standard_normal((cfg["T"], cfg["D"]))
    g = B.moe_backward(cfg, inp, dy)
    _, idx0 = _loss(cfg, inp, dy)
    assert np.array_equal(g["idx"], idx0)
    skipped = checked = 0
    for name in PARAMS:
        if inp.get(name) is None:
            assert g[GRAD_OF[name]] is None, name
            continue
        base = np.array(inp[name], dtype=np.float64)
        an = np.asarray(g[GRAD_OF[name]])
        assert an.shape == base.shape, name
        scale = 1.0 + float(np.max(np.abs(an)))
        for pos in np.ndindex(base.shape):
            vals = []
            flip = False
            for s in (+1, -1):
                p = base.copy()
                p[pos] += s * h
                q = dict(inp)
                q[name] = p
                L, idx = _loss(cfg, q, dy)
                flip |= not np.array_equal(idx, idx0)
                vals.append(L)
            if flip:
                skipped += 1
                continue
            fd = (vals[0] - vals[1]) / (2 * h)
            checked += 1
            assert abs(fd - an[pos]) <= 1e-6 * scale, (name, pos, fd, an[pos])
    assert skipped <= checked // 20, (skipped, checked)


def pin_fd_glam(B):
    _fd_check(B, BWD_TINY[0], 101)


def pin_fd_glm_shared(B):
    _fd_check(B, BWD_TINY[1], 102)


def pin_fd_softmax_unnormalised(B):
    _fd_check(B, BWD_TINY[2], 103)


def pin_fd_sigmoid_unnormalised(B):
    _fd_check(B, BWD_TINY[3], 104)


def pin_fd_grouped(B):
    _fd_check(B, BWD_TINY[4], 105)


def pin_softmax_shift_invariance(B):
    """Softmax weights do not change when the same constant is added to every
    logit of a token, so each token's logit gradient sums to zero."""
    for cfg in (BWD_TINY[0], BWD_TINY[2]):
        inp = tiny_inputs(cfg, 110)
        dy = np.random.default_rng(111).standard_normal((cfg["T"], cfg["D"]))
        dl = B.moe_backward(cfg, inp, dy)["dl"]
        assert np.allclose(dl.sum(axis=1), 0.0, atol=1e-13)
        assert np.abs(dl).max() > 1e-3


def pin_activation_derivatives(B):
    """The activation derivatives against a 5-point difference stencil of the
    library-pinned activations, far from any tiny-layer argument range."""
    v = np.linspace(-9, 9, 3601)
    h = 1e-3
    for f, df in ((FWD.gelu_tanh, B.gelu_tanh_grad), (FWD.silu, B.silu_grad)):
        fd = (-f(v + 2 * h) + 8 * f(v + h) - 8 * f(v - h) + f(v - 2 * h)) / (12 * h)
        assert np.allclose(df(v), fd, rtol=0, atol=1e-10)


def pin_expert_load(B):
    """Counts and coefficient of variation against a plain count and
    statistics.pstdev / statistics.mean."""
    rng = np.random.default_rng(7)
    M = 9
    idx = rng.integers(0, M + 1, size=(40, 3))     # value M = sentinel, not counted
    s = B.expert_load(idx, M)
    counts = [sum(1 for v in idx.reshape(-1).tolist() if v == e) for e in range(M)]
    assert s["counts"].tolist() == counts
    assert math.isclose(s["cv"], statistics.pstdev(counts) / statistics.mean(counts), rel_tol=1e-12)
    assert math.isclose(s["max_over_mean"], max(counts) / statistics.mean(counts), rel_tol=1e-12)


def pin_dense_backward(B):
    """The dense FFN layer's backward equals the layer backward of a single
    expert with weight one (M = 1, k = 1, renormalised softmax), whose
    gradients the finite-difference pins cover; and the dense layer's own
    input gradient against finite differences."""
    cfg = dict(T=4, D=5, M=1, k=1, gate="softmax", act="gelu_tanh", I=3,
               norm_topk_prob=1, alpha=1.0, eps=1e-20, I_sh=0)
    inp = tiny_inputs(cfg, 120)
    dy = np.random.default_rng(121).standard_normal((cfg["T"], cfg["D"]))
    d = B.dense_layer_backward(inp["x"], "gelu_tanh", inp["w1"][0], inp["w2"][0], inp["b1"][0],
                               inp["b2"][0], dy)
    h = 1e-5
    for pos in np.ndindex(inp["x"].shape):
        vals = []
        for s in (+1, -1):
            x = inp["x"].copy()
            x[pos] += s * h
            y = FWD.dense_layer(x, "gelu_tanh", inp["w1"][0], inp["w2"][0], inp["b1"][0], inp["b2"][0])
            vals.append(float(np.sum(dy * y)))
        assert abs((vals[0] - vals[1]) / (2 * h) - d["dx"][pos]) <= 1e-7
    g = B.moe_backward(cfg, inp, dy)
    assert np.allclose(g["dw1"][0], d["dw1"], rtol=1e-12, atol=1e-13)
    assert np.allclose(g["db2"][0], d["db2"], rtol=1e-12, atol=1e-13)


def pin_single_choice_sigmoid_router(B):
    """With one chosen expert the renormalised sigmoid weight is
    alpha g / (g + eps), constant to within eps ("Shared Expert" GLM-4.5
    note, eq. g-bar with k = 1), so the router gets no gradient: dlogits and
    dW_r are zero, and dx is that of the experts alone."""
    cfg = dict(T=7, D=5, M=4, k=1, gate="sigmoid_bias", act="swiglu", I=3,
               norm_topk_prob=1, alpha=2.5, eps=1e-20, I_sh=2)
    inp = tiny_inputs(cfg, 130)
    dy = np.random.default_rng(131).standard_normal((cfg["T"], cfg["D"]))
    g = B.moe_backward(cfg, inp, dy)
    assert np.abs(g["dl"]).max() <= 1e-12 and np.abs(g["dw_r"]).max() <= 1e-12
    assert np.abs(g["dw"]).max() > 1e-3


def pin_absolute_term_sums(B):
    """The absolute-term sums of the weight gradients (the scale of their
    rounding error), by a brute-force loop over the rows of each expert:
    dw1_abs[n, d] = sum_r |dpre[r, n]| |x[r, d]|, dw2_abs[d, i] =
    sum_r |dout[r, d]| |a[r, i]|, db1_abs[n] = sum_r |dpre[r, n]|, with
    dpre = dL/d(pre-activation) and dout the expert's upstream gradient,
    both from the finite-difference-pinned gradients above; and each sum
    bounds its gradient: |dw| <= dw_abs elementwise (triangle inequality)."""
    for cfg in (BWD_TINY[0], BWD_TINY[1]):
        inp = tiny_inputs(cfg, 140)
        dy = np.random.default_rng(141).standard_normal((cfg["T"], cfg["D"]))
        g = B.moe_backward(cfg, inp, dy)
        for name in ("dw1", "dw2", "db1", "dsh_w1", "dsh_w2", "dw_r"):
            if g[name] is not None:
                assert np.all(np.abs(g[name]) <= g[name + "_abs"] + 1e-12), name
        # the router's: dw_r_abs[d, m] = sum_t |x[t, d]| |dl[t, m]| by a scalar loop
        xa = np.abs(np.asarray(inp["x"], np.float64))
        for d, m in ((0, 0), (cfg["D"] - 1, cfg["M"] - 1), (1, 2)):
            s = 0.0
            for t in range(cfg["T"]):
                s += xa[t, d] * abs(g["dl"][t, m])
            assert abs(s - g["dw_r_abs"][d, m]) <= 1e-12 * max(1.0, s), (d, m)
        # brute force of one expert's sums from its own rows
        e = int(g["idx"][0, 0])
        tt, jj = np.nonzero(g["idx"] == e)
        x = np.asarray(inp["x"], np.float64)[tt]
        w1, w2 = np.asarray(inp["w1"][e], np.float64), np.asarray(inp["w2"][e], np.float64)
        dout = g["w"][tt, jj][:, None] * dy[tt]
        pre = x @ w1.T
        if cfg["act"] == "gelu_tanh":
            pre = pre + np.asarray(inp["b1"][e], np.float64)
            a = FWD.gelu_tanh(pre)
            dpre = (dout @ w2) * B.gelu_tanh_grad(pre)
        else:
            I = w1.shape[0] // 2
            a = FWD.silu(pre[:, :I]) * pre[:, I:]
            da = dout @ w2
            dpre = np.concatenate([da * pre[:, I:] * B.silu_grad(pre[:, :I]), da * FWD.silu(pre[:, :I])], axis=1)
        n1, D = w1.shape
        bf1 = np.zeros((n1, D))
        bf2 = np.zeros(w2.shape)
        for r in range(len(tt)):
            for n in range(n1):
                for d in range(D):
                    bf1[n, d] += abs(dpre[r, n]) * abs(x[r, d])
            for d in range(w2.shape[0]):
                for i in range(w2.shape[1]):
                    bf2[d, i] += abs(dout[r, d]) * abs(a[r, i])
        assert np.allclose(g["dw1_abs"][e], bf1, rtol=1e-12, atol=1e-14)
        assert np.allclose(g["dw2_abs"][e], bf2, rtol=1e-12, atol=1e-14)
        if g["db1_abs"] is not None:
            assert np.allclose(g["db1_abs"][e], np.abs(dpre).sum(axis=0), rtol=1e-12, atol=1e-14)


BWD_PINS = [
    pin_fd_glam, pin_fd_glm_shared, pin_fd_softmax_unnormalised, pin_fd_sigmoid_unnormalised,
    pin_fd_grouped, pin_softmax_shift_invariance, pin_activation_derivatives, pin_expert_load,
    pin_dense_backward, pin_single_choice_sigmoid_router, pin_absolute_term_sums,
]

"""Plain fp64 CPU oracle of the sparse Mixture-of-Experts FFN layer backward.

TEST INFRASTRUCTURE.  Only ``tests/`` and the benchmark's CPU legs may use
this module; the product path never does.  It shares no code with the CUDA
library.

The layer is the forward of ``moe_oracle`` (same pages, same readings).
Given the upstream gradient dy = dL/dy of a scalar loss L, this module
returns dL/d(every input): the tokens x, the router W_r, every routed
expert's weights and biases, and the shared expert's weights.  Each step is
the chain rule applied to one forward step, in the forward's notation:

  [GLaM]     "GLaM" note, section "Sparse MoE Layer": eq. FFN (the expert),
             eq. r_t (router), eq. S_t (top-k), eq. MoE (the weighted sum).
  [GLM45-SE] GLM-4.5 "Shared Expert" note, section "How it works": the
             sigmoid router with correction bias, eq. g-bar, w_i = alpha
             g-bar_i, E_sh, eq. y.
  [GLM5-SE]  "GLM-5 - Shared expert", section "All 5 steps" (SwiGLU).

Readings (the pages describe training only in prose):
  * The top-k choice S_t is a discrete function of the scores: its
    derivative is zero wherever it is defined, so the gradient flows only
    through the weights w_{t,j} of the experts already chosen and through
    the experts themselves.  The correction bias enters the choice only and
    so gets no gradient.  (The "GLM-4.5" note updates it outside the
    gradient, by load; the pages give no rule for that update.)
  * Training adds a penalty for uneven expert load (the "GLaM" industry
    article, section on the first route: the router is penalised for plans
    that load experts unevenly, and the load fluctuation fell by 40%).  The
    pages give no formula for the penalty, so this backward is that of the
    layer output alone; ``expert_load`` reports the load statistic itself:
    the tokens each expert receives and their coefficient of variation.

Pins: tests/oracle_pins_backward.py checks every gradient here against central finite
differences of the pinned forward oracle (an independent derivative), on
tiny layers of every router and expert variant, plus the shift invariance of
the renormalised softmax weights.
"""
from __future__ import annotations

import numpy as np

from . import moe_oracle as F

__all__ = ["gelu_tanh_grad", "silu_grad", "expert_ffn_backward", "router_backward",
           "moe_backward", "dense_layer_backward", "expert_load"]

_C = np.sqrt(2.0 / np.pi)
_A3 = 0.044715


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def gelu_tanh_grad(v):
    """d/dv of the tanh-form GELU: with u = c (v + a v^3),
    0.5 (1 + tanh u) + 0.5 v (1 - tanh^2 u) c (1 + 3 a v^2)."""
    v = _f64(v)
    th = np.tanh(_C * (v + _A3 * v ** 3))
    return 0.5 * (1.0 + th) + 0.5 * v * (1.0 - th * th) * _C * (1.0 + 3.0 * _A3 * v * v)


def silu_grad(v):
    """d/dv of v sigmoid(v) = sigmoid(v) (1 + v (1 - sigmoid(v)))."""
    v = _f64(v)
    s = F.sigmoid(v)
    return s * (1.0 + v * (1.0 - s))


def expert_ffn_backward(xe, act, w1e, w2e, b1e, b2e, dout):
    """Backward of one expert ([GLaM] eq. FFN, or the SwiGLU expert of
    [GLM5-SE]) on rows xe [n, D] with upstream gradient dout [n, D].

    Returns out (the forward value), dx [n, D], dw1 (shape of w1e), dw2
    (shape of w2e), db1, db2 (None when the bias is absent), and for the
    weight gradients the sums of the absolute values of their terms,
    dw1_abs = |dpre|^T |x|, dw2_abs = |dout|^T |a|, db1_abs = sum |dpre|:
    the scale of the rounding error of a sum whose terms carry a relative
    error (|fl(sum p_i) - sum p_i| <= u sum |p_i| when each p_i is off by
    at most u of itself)."""
    xe, w1e, w2e, dout = _f64(xe), _f64(w1e), _f64(w2e), _f64(dout)
    pre = xe @ w1e.T                                   # W1 x  [n, H] or [n, 2I]
    if act == "gelu_tanh":
        if b1e is not None:
            pre = pre + _f64(b1e)[None, :]
        a = F.gelu_tanh(pre)
    elif act == "swiglu":
        I = w1e.shape[0] // 2
        gate, up = pre[:, :I], pre[:, I:]
        a = F.silu(gate) * up
    else:
        raise ValueError(act)
    out = a @ w2e.T
    if b2e is not None:
        out = out + _f64(b2e)[None, :]
    dw2 = dout.T @ a                                   # d(W2 a)/dW2
    db2 = dout.sum(axis=0) if b2e is not None else None
    da = dout @ w2e
    if act == "gelu_tanh":
        dpre = da * gelu_tanh_grad(pre)
    else:
        dpre = np.concatenate([da * up * silu_grad(gate), da * F.silu(gate)], axis=1)
    db1 = dpre.sum(axis=0) if (act == "gelu_tanh" and b1e is not None) else None
    dw1 = dpre.T @ xe
    dx = dpre @ w1e
    return {"out": out, "dx": dx, "dw1": dw1, "dw2": dw2, "db1": db1, "db2": db2,
            "dw1_abs": np.abs(dpre).T @ np.abs(xe), "dw2_abs": np.abs(dout).T @ np.abs(a),
            "db1_abs": None if db1 is None else np.abs(dpre).sum(axis=0)}


def router_backward(idx, dw, logits, g, gate, norm_topk_prob, alpha, eps):
    """dL/d(logits) [T, M] from dL/dw [T, k] of the chosen experts'
    weights, through the weight formula of ``moe_oracle.topk_weights``.

    softmax, normalised: w_j = alpha q_j with q = softmax over S_t of the
      logits, so dl_i = alpha q_i (dw_i - sum_{j in S} q_j dw_j) for i in
      S_t, and 0 elsewhere.
    softmax, not normalised: w_j = alpha p_j with p the softmax over all M
      experts, so dl_i = alpha p_i ([i in S] dw_i - sum_{j in S} p_j dw_j)
      for every i.
    sigmoid_bias: w_j = alpha g_j / (G + eps) with G = sum_S g (or alpha
      g_j), so dg_i = alpha (dw_i / (G + eps) - sum_j dw_j g_j / (G + eps)^2)
      for i in S_t (alpha dw_i), and dl_i = dg_i g_i (1 - g_i).  The
      normalised form is evaluated centred, as
      alpha / (G + eps) * (dw_i - sum_j gbar_j dw_j) with gbar = g / (G + eps),
      the same value; with one chosen expert gbar is 1 to within eps, and
      the gradient (which is eps-small) comes out as 0 instead of the
      rounding residue of two equal terms.
    Chosen-expert indices equal to M (the sentinel) carry no weight."""
    idx = np.asarray(idx, dtype=np.int64)
    dw = _f64(dw)
    l = _f64(logits)
    T, M = l.shape
    dl = np.zeros((T, M))
    for t in range(T):
        S = [(j, int(e)) for j, e in enumerate(idx[t]) if e < M]
        if not S:
            continue
        js = np.array([j for j, _ in S])
        es = np.array([e for _, e in S])
        if gate == "softmax":
            if norm_topk_prob:
                ls = l[t, es]
                q = np.exp(ls - ls.max())
                q = q / q.sum()
                dl[t, es] = alpha * q * (dw[t, js] - np.dot(q, dw[t, js]))
            else:
                p = np.exp(l[t] - l[t].max())
                p = p / p.sum()
                ind = np.zeros(M)
                ind[es] = dw[t, js]
                dl[t] = alpha * p * (ind - np.dot(p[es], dw[t, js]))
        elif gate == "sigmoid_bias":
            gt = _f64(g)[t, es]
            if norm_topk_prob:
                den = gt.sum() + eps
                gbar = gt / den
                dg = alpha / den * (dw[t, js] - np.dot(gbar, dw[t, js]))
            else:
                dg = alpha * dw[t, js]
            dl[t, es] = dg * gt * (1.0 - gt)
        else:
            raise ValueError(gate)
    return dl


def moe_backward(cfg, inp, dy, idx=None):
    """Gradients of L = sum(dy * y) for the whole layer of
    ``moe_oracle.moe_forward`` (no addend: an added term only passes dy on).

    Returns dx [T, D], dw_r [D, M], dw1 / dw2 (stacked like w1 / w2),
    db1 / db2 (or None), dsh_w1 / dsh_w2 (or None), the intermediate
    dw [T, k] (gradient of each chosen weight) and dl [T, M] (of the
    logits), with the forward's routing, and the absolute-term sums
    (*_abs) of the expert and shared weight gradients (see
    expert_ffn_backward) and of the router's, dw_r_abs = |x|^T |dl|: the
    scale of the rounding error of a sum whose terms carry one bf16
    rounding of an operand (dl, when the router's backward GEMMs run on
    bf16 operands)."""
    r = F.route(inp["x"], inp["w_r"], inp.get("e_bias"), cfg["k"], cfg["gate"],
                cfg["norm_topk_prob"], cfg["alpha"], cfg["eps"], cfg.get("n_group", 1),
                cfg.get("topk_group", 1))
    if idx is not None:
        r["idx"] = np.asarray(idx, dtype=np.int64)
        r["w"] = F.topk_weights(r["idx"], r["logits"], r["g"], cfg["gate"], cfg["norm_topk_prob"],
                                cfg["alpha"], cfg["eps"])
    x = _f64(inp["x"])
    dy = _f64(dy)
    T, D = x.shape
    M, k = cfg["M"], cfg["k"]
    w1, w2 = _f64(inp["w1"]), _f64(inp["w2"])
    b1 = None if inp.get("b1") is None else _f64(inp["b1"])
    b2 = None if inp.get("b2") is None else _f64(inp["b2"])
    dx = np.zeros((T, D))
    dw1, dw2 = np.zeros_like(w1), np.zeros_like(w2)
    dw1_abs, dw2_abs = np.zeros_like(w1), np.zeros_like(w2)
    db1 = None if b1 is None else np.zeros_like(b1)
    db1_abs = None if b1 is None else np.zeros_like(b1)
    db2 = None if b2 is None else np.zeros_like(b2)
    dw = np.zeros((T, k))
    for e in range(M):
        tt, jj = np.nonzero(r["idx"] == e)
        if tt.size == 0:
            continue
        wr = r["w"][tt, jj][:, None]
        # y_t += w E_e(x_t): dE = w dy_t, dw = <dy_t, E_e(x_t)>
        g = expert_ffn_backward(x[tt], cfg["act"], w1[e], w2[e],
                                None if b1 is None else b1[e], None if b2 is None else b2[e], wr * dy[tt])
        dw[tt, jj] = np.sum(dy[tt] * g["out"], axis=1)
        np.add.at(dx, tt, g["dx"])
        dw1[e] += g["dw1"]
        dw2[e] += g["dw2"]
        dw1_abs[e] += g["dw1_abs"]
        dw2_abs[e] += g["dw2_abs"]
        if db1 is not None:
            db1[e] += g["db1"]
            db1_abs[e] += g["db1_abs"]
        if db2 is not None:
            db2[e] += g["db2"]
    dsh_w1 = dsh_w2 = dsh_w1_abs = dsh_w2_abs = None
    if cfg.get("I_sh"):
        gs = expert_ffn_backward(x, "swiglu", inp["sh_w1"], inp["sh_w2"], None, None, dy)
        dx += gs["dx"]
        dsh_w1, dsh_w2 = gs["dw1"], gs["dw2"]
        dsh_w1_abs, dsh_w2_abs = gs["dw1_abs"], gs["dw2_abs"]
    dl = router_backward(r["idx"], dw, r["logits"], r["g"], cfg["gate"], cfg["norm_topk_prob"],
                         cfg["alpha"], cfg["eps"])
    w_r = _f64(inp["w_r"])
    dx += dl @ w_r.T                                   # logits = x W_r
    dw_r = x.T @ dl
    return {"dx": dx, "dw_r": dw_r, "dw1": dw1, "dw2": dw2, "db1": db1, "db2": db2,
            "dsh_w1": dsh_w1, "dsh_w2": dsh_w2, "dw": dw, "dl": dl, "idx": r["idx"], "w": r["w"],
            "dw1_abs": dw1_abs, "dw2_abs": dw2_abs, "db1_abs": db1_abs, "dsh_w1_abs": dsh_w1_abs,
            "dsh_w2_abs": dsh_w2_abs, "dw_r_abs": np.abs(x).T @ np.abs(dl)}


def dense_layer_backward(x, act, w1, w2, b1, b2, dy):
    """Backward of ``moe_oracle.dense_layer`` (the dense FFN between sparse
    layers): the expert backward on every token with dout = dy."""
    return expert_ffn_backward(x, act, w1, w2, b1, b2, dy)


def expert_load(idx, M):
    """Load statistic of one routing: tokens per expert (sentinel pairs not
    counted), their mean, and the coefficient of variation std / mean (the
    "fluctuation" of expert load the GLaM article reports training reduced)."""
    idx = np.asarray(idx, dtype=np.int64).reshape(-1)
    counts = np.bincount(idx[idx < M], minlength=M).astype(np.int64)
    mean = counts.mean() if M else 0.0
    cv = float(counts.std() / mean) if mean > 0 else 0.0
    return {"counts": counts, "mean": float(mean), "cv": cv,
            "max_over_mean": float(counts.max() / mean) if mean > 0 else 0.0}

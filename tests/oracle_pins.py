"""Checks that pin the CPU oracle to facts outside its own code.

Each ``pin_*`` function takes the oracle module and raises AssertionError if
the oracle disagrees with the fact it checks.  tests/test_oracle_pins.py runs
them on the real oracle; tests/test_oracle_mutations.py plants mistakes in a
patched oracle and checks that some pin catches each one.

The independent sides used here are:
  * library routines: torch.nn.functional.gelu(approximate="tanh"), silu,
    sigmoid, softmax, torch.nn.Linear;
  * closed forms from the pages: the renormalised top-2 softmax weight
    1 / (1 + exp(l2 - l1)) ("GLaM", eq. MoE), the sum of the sigmoid router's
    weights alpha * S / (S + eps) ("Shared Expert" GLM-4.5 note, eq. g-bar
    and w_i = alpha g-bar_i), the printed parameter counts ("GLM-5 - Shared
    expert", "Exact per-instance accounting");
  * brute force on tiny inputs: a per-token loop over ALL M experts with a
    0/1 mask from a full sort, written with Python scalars and torch.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split()
            vals[k] = float(v) if ("." in v or "e" in v) else int(v)
    return vals


def _t(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float64))


# ---------------------------------------------------------------------------
# activations against library routines
# ---------------------------------------------------------------------------

def pin_gelu(O):
    v = np.linspace(-8, 8, 4001)
    ref = F.gelu(_t(v), approximate="tanh").numpy()
    assert np.allclose(O.gelu_tanh(v), ref, rtol=1e-14, atol=1e-15)


def pin_silu_sigmoid(O):
    v = np.linspace(-30, 30, 6001)
    assert np.allclose(O.sigmoid(v), torch.sigmoid(_t(v)).numpy(), rtol=1e-14, atol=0)
    assert np.allclose(O.silu(v), F.silu(_t(v)).numpy(), rtol=1e-13, atol=1e-300)


# ---------------------------------------------------------------------------
# router
# ---------------------------------------------------------------------------

def _brute_topk(scores, k):
    out = []
    for row in scores:
        order = sorted(range(len(row)), key=lambda e: (-float(row[e]), e))
        out.append(order[:k])
    return np.array(out, dtype=np.int64)


def pin_topk_bruteforce(O):
    rng = np.random.default_rng(1)
    for M, k in [(8, 2), (16, 4), (33, 8), (5, 5), (1, 1)]:
        s = rng.integers(-4, 5, size=(64, M)).astype(np.float64) * 0.25  # many exact ties
        assert np.array_equal(O.topk_select(s, k), _brute_topk(s, k)), (M, k)
        s = rng.standard_normal((64, M))
        assert np.array_equal(O.topk_select(s, k), _brute_topk(s, k)), (M, k)


def pin_softmax_top2_closed_form(O):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((40, 16))
    w_r = rng.standard_normal((16, 8)) * 0.3
    r = O.route(x, w_r, None, 2, "softmax", 1, 1.0, 1e-20)
    logits = x @ w_r
    for t in range(40):
        e1, e2 = r["idx"][t]
        l1, l2 = logits[t, e1], logits[t, e2]
        a1 = 1.0 / (1.0 + math.exp(l2 - l1))
        assert abs(r["w"][t, 0] - a1) < 1e-14 and abs(r["w"][t, 1] - (1 - a1)) < 1e-14
    # the renormalised weights equal the library softmax renormalised over S
    p = torch.softmax(_t(logits), dim=1).numpy()
    ps = np.take_along_axis(p, r["idx"], axis=1)
    assert np.allclose(r["w"], ps / ps.sum(1, keepdims=True), rtol=1e-13)
    # without renormalisation: the full softmax probabilities
    r2 = O.route(x, w_r, None, 2, "softmax", 0, 1.0, 1e-20)
    assert np.allclose(r2["w"], ps, rtol=1e-13)


def pin_sigmoid_router(O):
    rng = np.random.default_rng(3)
    T, D, M, k, alpha, eps = 50, 24, 16, 4, 2.5, 1e-20
    x = rng.standard_normal((T, D))
    w_r = rng.standard_normal((D, M)) * 0.3
    bias = rng.uniform(-0.1, 0.1, M)
    r = O.route(x, w_r, bias, k, "sigmoid_bias", 1, alpha, eps)
    g = torch.sigmoid(_t(x @ w_r)).numpy()
    # selection over g + bias (brute force), weights from unbiased g
    assert np.array_equal(r["idx"], _brute_topk(g + bias[None, :], k))
    gs = np.take_along_axis(g, r["idx"], axis=1)
    S = gs.sum(1)
    assert np.allclose(r["w"].sum(1), alpha * S / (S + eps), rtol=1e-14)
    assert np.allclose(r["w"], alpha * gs / S[:, None], rtol=1e-13)
    # without renormalisation the weights are alpha * g
    r2 = O.route(x, w_r, bias, k, "sigmoid_bias", 0, alpha, eps)
    assert np.allclose(r2["w"], alpha * gs, rtol=1e-14)


def pin_bias_selects_only(O):
    """A large correction bias forces an expert into S, but its weight still
    comes from the unbiased sigmoid score ("Shared Expert" GLM-4.5 note:
    the top-8 after the bias, then "those 8 sigmoid scores g_i")."""
    rng = np.random.default_rng(4)
    T, D, M, k = 20, 8, 6, 2
    x = rng.standard_normal((T, D))
    w_r = rng.standard_normal((D, M))
    bias = np.zeros(M)
    bias[3] = 10.0
    r = O.route(x, w_r, bias, k, "sigmoid_bias", 1, 1.0, 1e-20)
    assert (r["idx"][:, 0] == 3).all()
    g = torch.sigmoid(_t(x @ w_r)).numpy()
    gs = np.take_along_axis(g, r["idx"], axis=1)
    assert np.allclose(r["w"], gs / gs.sum(1, keepdims=True), rtol=1e-13)


def _brute_group_topk(s, k, n_group, topk_group):
    """Group-limited top-k with Python scalars: group score = sum of the two
    largest member scores, the topk_group best groups (lower index on ties),
    then the k best eligible experts (lower index on ties)."""
    T, M = s.shape
    size = M // n_group
    out = np.zeros((T, k), dtype=np.int64)
    for t in range(T):
        row = [float(v) for v in s[t]]
        gscore = []
        for gi in range(n_group):
            members = sorted(row[gi * size:(gi + 1) * size], reverse=True)
            gscore.append(sum(members[:2]))
        groups = sorted(range(n_group), key=lambda gi: (-gscore[gi], gi))[:topk_group]
        eligible = [e for e in range(M) if e // size in groups]
        best = sorted(eligible, key=lambda e: (-row[e], e))[:k]
        out[t] = best
    return out


def pin_group_limit(O):
    """Group-limited routing ("Shared Expert" GLM-4.5 note: the router
    "optionally masks by expert group") against a scalar brute force, and the
    two groupings that must reduce to the plain top-k."""
    rng = np.random.default_rng(11)
    for M, n_group, topk_group, k in [(8, 4, 2, 3), (12, 4, 2, 4), (12, 3, 1, 2), (16, 8, 3, 5),
                                      (6, 6, 2, 2)]:
        for s in (rng.standard_normal((48, M)) - 0.5,                            # negative scores too
                  rng.integers(-3, 4, size=(48, M)).astype(np.float64) * 0.5):  # many exact ties
            got = O.topk_select(O.group_limit(s, n_group, topk_group), k)
            assert np.array_equal(got, _brute_group_topk(s, k, n_group, topk_group)), (M, n_group)
    s = rng.standard_normal((64, 16))
    plain = _brute_topk(s, 4)
    assert np.array_equal(O.topk_select(O.group_limit(s, 4, 4), 4), plain)    # every group kept
    assert np.array_equal(O.topk_select(O.group_limit(s, 16, 4), 4), plain)   # one expert per group
    assert np.array_equal(O.topk_select(O.group_limit(s, 1, 1), 4), plain)    # no grouping
    # through the router: selection masked by group, weights from the gate values
    x = rng.standard_normal((30, 12))
    w_r = rng.standard_normal((12, 16)) * 0.4
    bias = rng.uniform(-0.3, 0.1, 16)
    r = O.route(x, w_r, bias, 4, "sigmoid_bias", 1, 2.5, 1e-20, 4, 2)
    g = torch.sigmoid(_t(x @ w_r)).numpy()
    assert np.array_equal(r["idx"], _brute_group_topk(g + bias[None, :], 4, 4, 2))
    gs = np.take_along_axis(g, r["idx"], axis=1)
    assert np.allclose(r["w"], 2.5 * gs / gs.sum(1, keepdims=True), rtol=1e-13)


# ---------------------------------------------------------------------------
# dispatch
# ---------------------------------------------------------------------------

def pin_sentinel(O):
    """Index M is the "no expert" class ("GLM-5 - Shared expert", the quoted
    GlmMoeDsaExperts.forward: one_hot over M + 1 classes, class M skipped):
    a pair holding it is dispatched nowhere and contributes nothing."""
    rng = np.random.default_rng(8)
    T, k, M = 23, 3, 6
    idx = np.stack([rng.choice(M, size=k, replace=False) for _ in range(T)])
    drop = rng.random((T, k)) < 0.3
    idx_s = np.where(drop, M, idx)
    w = rng.random((T, k))
    p = O.permute(idx_s, w, M)
    assert p["counts"].sum() == (~drop).sum() == p["offsets"][M]
    assert (p["slot_of"][drop] == -1).all()
    s = 0
    for e in range(M):
        for j in range(k):
            for t in range(T):
                if idx_s[t, j] == e:
                    assert p["slot_of"][t, j] == s and p["row_token"][s] == t
                    s += 1
    # contribution: the sentinel pairs add nothing, i.e. the same as weight 0
    cfg = dict(TINY[2])
    inp = tiny_inputs(cfg, 70)
    r = O.route(inp["x"], inp["w_r"], inp["e_bias"], cfg["k"], cfg["gate"], 1, cfg["alpha"], cfg["eps"])
    dropk = np.zeros_like(r["idx"], dtype=bool)
    dropk[::2, 1] = True
    idx2 = np.where(dropk, cfg["M"], r["idx"])
    w0 = np.where(dropk, 0.0, r["w"])

    def get(e):
        return inp["w1"][e], inp["w2"][e], None, None
    y_s = O.moe_tokens(inp["x"], idx2, r["w"], cfg["act"], get, None, sentinel=cfg["M"])
    y_0 = O.moe_tokens(inp["x"], r["idx"], w0, cfg["act"], get, None)
    assert np.allclose(y_s, y_0, rtol=1e-13, atol=1e-13)


def pin_forward_sentinel(O):
    """The whole-layer oracle given a selection that holds the sentinel M:
    each token's output is, by a per-pair loop over its kept pairs only,
    sum_j w[t, j] E_idx[t, j](x_t) plus the shared expert; a token whose
    pairs are all sentinels gets the shared expert alone."""
    cfg = dict(TINY[2])
    inp = tiny_inputs(cfg, 71)
    r = O.route(inp["x"], inp["w_r"], inp["e_bias"], cfg["k"], cfg["gate"], 1, cfg["alpha"], cfg["eps"])
    M = cfg["M"]
    idx = r["idx"].copy()
    idx[1::3, 0] = M
    idx[4, :] = M
    out = O.moe_forward(cfg, inp, idx=idx, w=r["w"])
    assert out["offsets"][M] == (idx < M).sum()
    for t in range(cfg["T"]):
        ref = np.zeros(cfg["D"])
        for j in range(cfg["k"]):
            e = idx[t, j]
            if e == M:
                continue
            h = inp["w1"][e] @ inp["x"][t]
            I = h.shape[0] // 2
            a = (h[:I] / (1.0 + np.exp(-h[:I]))) * h[I:]
            ref += r["w"][t, j] * (inp["w2"][e] @ a)
        if cfg.get("I_sh"):
            hs = inp["sh_w1"] @ inp["x"][t]
            Is = hs.shape[0] // 2
            ref += inp["sh_w2"] @ ((hs[:Is] / (1.0 + np.exp(-hs[:Is]))) * hs[Is:])
        assert np.allclose(out["y"][t], ref, rtol=1e-12, atol=1e-12), t
    try:
        O.moe_forward(cfg, inp, idx=idx)
    except ValueError:
        pass
    else:
        raise AssertionError("a sentinel selection without weights must be refused")


def pin_permute(O):
    rng = np.random.default_rng(5)
    for T, k, M in [(37, 3, 7), (64, 8, 16), (1, 1, 1), (5, 4, 64)]:
        idx = np.stack([rng.choice(M, size=k, replace=False) for _ in range(T)])
        w = rng.random((T, k))
        p = O.permute(idx, w, M)
        assert p["counts"].sum() == T * k
        assert np.array_equal(p["offsets"][1:] - p["offsets"][:-1], p["counts"])
        # brute force enumeration: expert by expert, slot j, then token t
        s = 0
        for e in range(M):
            assert p["offsets"][e] == s
            for j in range(k):
                for t in range(T):
                    if idx[t, j] == e:
                        assert p["slot_of"][t, j] == s
                        assert p["row_token"][s] == t
                        assert p["row_w"][s] == w[t, j]
                        s += 1
        assert s == T * k
        assert sorted(p["slot_of"].reshape(-1).tolist()) == list(range(T * k))


# ---------------------------------------------------------------------------
# experts and the whole layer
# ---------------------------------------------------------------------------

def _lib_ffn(xt, act, w1e, w2e, b1e, b2e):
    """One expert on one token with torch library layers (fp64)."""
    xt = _t(xt)[None, :]
    if act == "gelu_tanh":
        l1 = torch.nn.Linear(w1e.shape[1], w1e.shape[0], bias=b1e is not None).double()
        l2 = torch.nn.Linear(w2e.shape[1], w2e.shape[0], bias=b2e is not None).double()
        with torch.no_grad():
            l1.weight.copy_(_t(w1e))
            l2.weight.copy_(_t(w2e))
            if b1e is not None:
                l1.bias.copy_(_t(b1e))
            if b2e is not None:
                l2.bias.copy_(_t(b2e))
            return l2(F.gelu(l1(xt), approximate="tanh"))[0].numpy()
    I = w1e.shape[0] // 2
    gate = torch.nn.Linear(w1e.shape[1], I, bias=False).double()
    up = torch.nn.Linear(w1e.shape[1], I, bias=False).double()
    down = torch.nn.Linear(I, w2e.shape[0], bias=False).double()
    with torch.no_grad():
        gate.weight.copy_(_t(w1e[:I]))
        up.weight.copy_(_t(w1e[I:]))
        down.weight.copy_(_t(w2e))
        return down(F.silu(gate(xt)) * up(xt))[0].numpy()


def brute_force_forward(cfg, inp):
    """Per token: score all M experts, full sort, 0/1 mask, run ALL experts
    through library layers, y_t = sum_e mask_e w_e E_e(x_t) (+ E_sh(x_t))."""
    x = np.asarray(inp["x"], np.float64)
    w_r = np.asarray(inp["w_r"], np.float64)
    T, M, k = x.shape[0], cfg["M"], cfg["k"]
    bias = inp.get("e_bias")
    y = np.zeros_like(x)
    for t in range(T):
        logit = [float(np.dot(x[t], w_r[:, e])) for e in range(M)]
        if cfg["gate"] == "softmax":
            sel = logit
        else:
            g = [1.0 / (1.0 + math.exp(-l)) for l in logit]
            sel = [g[e] + (0.0 if bias is None else float(bias[e])) for e in range(M)]
        chosen = sorted(range(M), key=lambda e: (-sel[e], e))[:k]
        if cfg["gate"] == "softmax":
            if cfg["norm_topk_prob"]:
                ex = [math.exp(logit[e] - logit[chosen[0]]) for e in chosen]
                wts = [v / sum(ex) for v in ex]
            else:
                full = [math.exp(l - max(logit)) for l in logit]
                wts = [full[e] / sum(full) for e in chosen]
        else:
            gs = [g[e] for e in chosen]
            wts = [v / (sum(gs) + cfg["eps"]) for v in gs] if cfg["norm_topk_prob"] else gs
        mask = [0.0] * M
        for e, v in zip(chosen, wts):
            mask[e] = cfg["alpha"] * v
        for e in range(M):
            b1 = None if inp.get("b1") is None else inp["b1"][e]
            b2 = None if inp.get("b2") is None else inp["b2"][e]
            y[t] += mask[e] * _lib_ffn(x[t], cfg["act"], inp["w1"][e], inp["w2"][e], b1, b2)
        if cfg.get("I_sh"):
            y[t] += _lib_ffn(x[t], "swiglu", inp["sh_w1"], inp["sh_w2"], None, None)
    return y


def tiny_inputs(cfg, seed):
    rng = np.random.default_rng(seed)
    T, D, M, I = cfg["T"], cfg["D"], cfg["M"], cfg["I"]
    n1 = 2 * I if cfg["act"] == "swiglu" else I
    inp = {
        "x": rng.standard_normal((T, D)),
        "w_r": rng.standard_normal((D, M)) * 0.5,
        "e_bias": rng.uniform(-0.1, 0.1, M) if cfg["gate"] == "sigmoid_bias" else None,
        "w1": rng.standard_normal((M, n1, D)) / math.sqrt(D),
        "w2": rng.standard_normal((M, D, I)) / math.sqrt(I),
        "b1": rng.standard_normal((M, I)) * 0.1 if cfg["act"] == "gelu_tanh" else None,
        "b2": rng.standard_normal((M, D)) * 0.1 if cfg["act"] == "gelu_tanh" else None,
    }
    if cfg.get("I_sh"):
        inp["sh_w1"] = rng.standard_normal((2 * cfg["I_sh"], D)) / math.sqrt(D)
        inp["sh_w2"] = rng.standard_normal((D, cfg["I_sh"])) / math.sqrt(cfg["I_sh"])
    return inp


TINY = [
    dict(T=12, D=16, M=8, k=2, gate="softmax", act="gelu_tanh", I=24,
         norm_topk_prob=1, alpha=1.0, eps=1e-20, I_sh=0),
    dict(T=10, D=16, M=6, k=3, gate="softmax", act="gelu_tanh", I=8,
         norm_topk_prob=0, alpha=1.0, eps=1e-20, I_sh=0),
    dict(T=9, D=16, M=16, k=4, gate="sigmoid_bias", act="swiglu", I=12,
         norm_topk_prob=1, alpha=2.5, eps=1e-20, I_sh=12),
    dict(T=7, D=8, M=5, k=5, gate="sigmoid_bias", act="swiglu", I=4,
         norm_topk_prob=0, alpha=1.0, eps=1e-20, I_sh=8),
]


def pin_bruteforce_forward(O):
    for n, cfg in enumerate(TINY):
        inp = tiny_inputs(cfg, 10 + n)
        y = O.moe_forward(cfg, inp)["y"]
        yb = brute_force_forward(cfg, inp)
        assert np.allclose(y, yb, rtol=1e-12, atol=1e-12), n


def pin_single_expert_is_dense_ffn(O):
    """M = 1, k = 1 reduces the layer to one dense FFN ("GLaM", eq. FFN),
    checked against torch.nn.Linear + library GELU / SiLU."""
    for act in ("gelu_tanh", "swiglu"):
        cfg = dict(T=6, D=12, M=1, k=1, gate="softmax", act=act, I=20,
                   norm_topk_prob=1, alpha=1.0, eps=1e-20, I_sh=0)
        inp = tiny_inputs(cfg, 30)
        y = O.moe_forward(cfg, inp)["y"]
        for t in range(cfg["T"]):
            b1 = None if inp["b1"] is None else inp["b1"][0]
            b2 = None if inp["b2"] is None else inp["b2"][0]
            ref = _lib_ffn(inp["x"][t], act, inp["w1"][0], inp["w2"][0], b1, b2)
            assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-13), act


def pin_k_equals_m(O):
    """k = M with renormalised softmax gates: every expert weighted by its
    full softmax probability (torch.softmax)."""
    cfg = dict(T=5, D=10, M=4, k=4, gate="softmax", act="gelu_tanh", I=6,
               norm_topk_prob=1, alpha=1.0, eps=1e-20, I_sh=0)
    inp = tiny_inputs(cfg, 40)
    y = O.moe_forward(cfg, inp)["y"]
    p = torch.softmax(_t(inp["x"] @ inp["w_r"]), dim=1).numpy()
    for t in range(cfg["T"]):
        ref = sum(p[t, e] * _lib_ffn(inp["x"][t], "gelu_tanh", inp["w1"][e], inp["w2"][e],
                                     inp["b1"][e], inp["b2"][e]) for e in range(4))
        assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-13)


def pin_shared_branch(O):
    """The shared expert reads the pre-routing x and is summed ("Shared
    Expert" GLM-4.5 note: E_sh is a function of x, not of the mixture):
    with alpha = 0 the layer is exactly E_sh(x), whatever the router."""
    cfg = dict(TINY[2])
    cfg["alpha"] = 0.0
    inp = tiny_inputs(cfg, 50)
    y0 = O.moe_forward(cfg, inp)["y"]
    inp2 = dict(inp)
    inp2["w_r"] = inp["w_r"][:, ::-1].copy() * 3.0
    inp2["e_bias"] = -inp["e_bias"]
    y1 = O.moe_forward(cfg, inp2)["y"]
    assert np.array_equal(y0, y1)
    for t in range(cfg["T"]):
        ref = _lib_ffn(inp["x"][t], "swiglu", inp["sh_w1"], inp["sh_w2"], None, None)
        assert np.allclose(y0[t], ref, rtol=1e-12, atol=1e-13)


def pin_sum_no_residual(O):
    """y is a sum with no residual inside the layer: zero weights give y = 0."""
    cfg = dict(TINY[2])
    inp = tiny_inputs(cfg, 60)
    for key in ("w1", "w2", "sh_w1", "sh_w2"):
        inp[key] = np.zeros_like(inp[key])
    y = O.moe_forward(cfg, inp)["y"]
    assert np.array_equal(y, np.zeros_like(y))
    # the block sum adds the other term outside the layer: with zero experts it is all that is left
    a = np.random.default_rng(13).standard_normal(np.asarray(inp["x"]).shape)
    assert np.array_equal(O.moe_forward(cfg, inp, addend=a)["y"], a)


def pin_dense_layer(O):
    """The dense FFN layer and the block sum ("GLaM" note, "Interleaving
    Dense and Sparse Layers": h^{l+1} = Attention(h^l) + DenseFFN(h^l))
    against torch.nn.functional.linear and the library activations."""
    rng = np.random.default_rng(12)
    T, D, I = 9, 12, 20
    x = rng.standard_normal((T, D))
    a = rng.standard_normal((T, D))
    w1 = rng.standard_normal((I, D)) * 0.3
    b1 = rng.standard_normal(I) * 0.1
    w2 = rng.standard_normal((D, I)) * 0.3
    b2 = rng.standard_normal(D) * 0.1
    ref = (_t(a) + F.linear(F.gelu(F.linear(_t(x), _t(w1), _t(b1)), approximate="tanh"), _t(w2), _t(b2))).numpy()
    assert np.allclose(O.dense_layer(x, "gelu_tanh", w1, w2, b1, b2, addend=a), ref, rtol=1e-12, atol=1e-12)
    wgu = rng.standard_normal((2 * I, D)) * 0.3
    ref = F.linear(F.silu(F.linear(_t(x), _t(wgu[:I]))) * F.linear(_t(x), _t(wgu[I:])), _t(w2)).numpy()
    assert np.allclose(O.dense_layer(x, "swiglu", wgu, w2), ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(O.dense_layer(x, "swiglu", wgu, w2, addend=a), ref + a, rtol=1e-12, atol=1e-12)


def pin_param_counts(O):
    g = read_golden("glm5_shared_expert_params.txt")
    D, W, L = g["hidden_size"], g["shared_width"], g["moe_blocks"]
    shared_only = O.param_count(D, 0, 0, "swiglu", I_sh=W, router=False)
    assert shared_only == g["per_instance_total"]
    assert shared_only == g["gate_projection"] + g["up_projection"] + g["down_projection"]
    assert L * shared_only == g["across_moe_blocks"]
    # 19,200 correction-bias values over 75 blocks -> 256 routed experts
    M = g["router_bias_values"] // L
    assert M * L == g["router_bias_values"]
    bias_only = O.param_count(D, M, 0, "swiglu", router=False, e_bias=True)
    assert bias_only * L == g["router_bias_values"]
    s = read_golden("glm45_shapes.txt")
    one_expert = O.param_count(s["hidden_size"], 1, s["moe_intermediate_size"], "swiglu", router=False)
    assert one_expert == 3 * 5120 * 1536 == 23592960


def pin_error_metrics(O):
    y_ref = np.array([[1.0, -2.0], [3.0, -4.0]])
    m = O.error_metrics(y_ref * 1.01, y_ref)
    assert abs(m["mean_rel"] - 0.01) < 1e-15
    rms = math.sqrt((1 + 4 + 9 + 16) / 4)
    assert abs(m["max_over_rms"] - 0.04 / rms) < 1e-15


def pin_adopt_topk(O):
    sel = np.array([[0.9, 0.5, 0.5 + 1e-7, 0.1], [0.9, 0.8, 0.7, 0.6]])
    ok, n, _ = O.adopt_topk(np.array([[0, 2], [0, 1]]), sel)
    assert ok and n == 0
    ok, n, _ = O.adopt_topk(np.array([[0, 1], [0, 1]]), sel)   # near-tie swap
    assert ok and n == 1
    ok, _, bad = O.adopt_topk(np.array([[0, 2], [0, 2]]), sel)  # real difference
    assert not ok and bad == 1
    ok, _, _ = O.adopt_topk(np.array([[2, 2], [0, 1]]), sel)   # duplicate index
    assert not ok


def pin_capacity_drop(O):
    """Expert capacity against a scalar loop over the (slot, token) order:
    a per-expert counter admits a pair while it is below the capacity.
    Invariants: kept counts never exceed it, an ample capacity drops nothing,
    a zero capacity drops everything, sentinels in the input stay."""
    rng = np.random.default_rng(21)
    for T, k, M in ((40, 2, 5), (33, 4, 8), (7, 3, 3)):
        idx = np.stack([rng.choice(M, size=k, replace=False) for _ in range(T)])
        idx[rng.random(idx.shape) < 0.1] = M
        for cap in (0, 1, 3, (T * k) // M, T * k):
            ref = idx.copy()
            seen = [0] * M
            for j in range(k):
                for t in range(T):
                    e = int(idx[t, j])
                    if e == M:
                        continue
                    if seen[e] >= cap:
                        ref[t, j] = M
                    else:
                        seen[e] += 1
            got = O.capacity_drop(idx, M, cap)
            assert np.array_equal(got, ref), (T, k, M, cap)
            kept = got[got < M]
            assert (np.bincount(kept, minlength=M) <= cap).all()
        assert np.array_equal(O.capacity_drop(idx, M, T * k), idx)
        assert (O.capacity_drop(idx, M, 0) == M).all()
    assert O.expert_capacity(1.0, 8192, 2, 64) == 256
    assert O.expert_capacity(1.25, 300, 4, 16) == 94
    assert O.expert_capacity(0.0, 300, 4, 16) == 0


ALL_PINS = [
    pin_gelu, pin_silu_sigmoid, pin_topk_bruteforce, pin_softmax_top2_closed_form,
    pin_sigmoid_router, pin_bias_selects_only, pin_group_limit, pin_permute, pin_sentinel, pin_forward_sentinel, pin_bruteforce_forward,
    pin_single_expert_is_dense_ffn, pin_k_equals_m, pin_shared_branch,
    pin_sum_no_residual, pin_dense_layer, pin_param_counts, pin_error_metrics, pin_adopt_topk,
    pin_capacity_drop,
]

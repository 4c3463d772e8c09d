"""Plain fp64 CPU oracle of the sparse Mixture-of-Experts FFN layer forward.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU legs may use this module; the product path never does.  It
shares no code with the CUDA library.

Inputs are the exact (bf16- or fp32-rounded) values the GPU sees, widened to
fp64; every step below runs in fp64 with NumPy.  Each function follows one
passage of the source pages, cited by page title and section/equation:

  [GLaM]     "GLaM" architecture note, section "Sparse MoE Layer"
             (eq. FFN, eq. r_t, eq. S_t, eq. MoE).
  [GLM45-SE] "Shared Expert" study note for GLM-4.5, section "How it works"
             (E_sh, the sigmoid router with correction bias, eq. g-bar,
             w_i = alpha g-bar_i, eq. y).
  [GLM5-SE]  "GLM-5 - Shared expert" (OpenModelAtlas), sections "All 5 steps",
             "Exact per-instance accounting" and the quoted
             GlmMoeDsaExperts / GlmMoeDsaMoE / GlmMoeDsaMLP forward excerpts.

Readings taken where the pages leave a step open:
  * GLaM's "normalized gate weight": the softmax probabilities of the k
    selected experts renormalised to sum to one; because the full softmax
    denominator cancels, alpha_j = exp(l_j - l_max) / sum_S exp(l - l_max).
  * GLaM's sigma: GELU with the tanh approximation.
  * The correction bias enters the selection only; weights use the unbiased
    sigmoid scores g_i.
  * Selection order: descending score, exact ties to the lower expert index;
    slot j of a token is its j-th largest score.
  * Dispatch order inside an expert's segment: by (slot j, then token t),
    the order the quoted GlmMoeDsaExperts.forward enumerates with
    ``torch.where`` over the [k, T] expert mask.
  * The routed weight multiplies b2 too: w * (W2 h + b2).
  * Group-limited routing ([GLM45-SE]: the router "optionally masks by
    expert group"; the note gives no rule): the M experts form n_group equal
    groups of consecutive indices; a group scores the sum of its two largest
    selection scores (its only score when a group holds one expert); the
    topk_group best groups (ties to the lower group index) stay eligible and
    every other expert is excluded from the top-k.  n_group = 1 is no mask.
  * Expert capacity (no page gives a rule): expert e keeps the first
    ceil(factor T k / M) of its pairs in the dispatch order above and the
    rest become the sentinel below; weights are not renormalised.
  * Expert index M (one past the last expert) is the "no expert" sentinel of
    the quoted GlmMoeDsaExperts.forward (one_hot over M + 1 classes, class M
    skipped): such a (token, slot) pair is dispatched nowhere and adds
    nothing to y.

Pins: every function here is checked, independently of its own code, by
tests/test_oracle_pins.py (library routines, closed forms, invariants, brute
force over all experts on tiny inputs, and the parameter counts the GLM-5 page
prints).  The pages print no worked example of a layer output, so full-size
outputs rest on this definition plus those pins.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "gelu_tanh", "silu", "sigmoid", "router_logits", "selection_scores",
    "topk_select", "group_limit", "topk_weights", "route", "permute", "expert_capacity", "capacity_drop",
    "expert_ffn",
    "shared_expert", "moe_tokens", "moe_forward", "dense_layer", "adopt_topk",
    "param_count", "error_metrics",
]


def _f64(a):
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# Activations
# ---------------------------------------------------------------------------

def gelu_tanh(v):
    """sigma of [GLaM] eq. FFN, read as GELU with the tanh approximation:
    0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3)))."""
    v = _f64(v)
    return 0.5 * v * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (v + 0.044715 * v ** 3)))


def sigmoid(v):
    v = _f64(v)
    return 1.0 / (1.0 + np.exp(-v))


def silu(v):
    """[GLM5-SE] "All 5 steps": a = g * sigmoid(g)."""
    v = _f64(v)
    return v * sigmoid(v)


# ---------------------------------------------------------------------------
# Router
# ---------------------------------------------------------------------------

def router_logits(x, w_r):
    """Raw router scores W_r x_t for every token ([GLaM] eq. r_t before the
    softmax; [GLM45-SE] "a sigmoid router scores the routed experts").
    x is [T, D]; w_r is stored [D, M], so the scores are x @ w_r."""
    return _f64(x) @ _f64(w_r)


def selection_scores(logits, gate, e_bias=None):
    """Scores the top-k is taken over, and the gate values the weights use.

    softmax ([GLaM] eq. r_t, eq. S_t): the top-k of softmax(l) is the top-k
    of l (softmax is monotone), so the selection score is the logit itself.
    sigmoid_bias ([GLM45-SE]): g = sigmoid(l); selection score g + e_bias.
    Returns (selection score [T, M], gate value [T, M])."""
    logits = _f64(logits)
    if gate == "softmax":
        return logits, logits
    if gate == "sigmoid_bias":
        g = sigmoid(logits)
        b = np.zeros(logits.shape[1]) if e_bias is None else _f64(e_bias)
        return g + b[None, :], g
    raise ValueError(gate)


def topk_select(sel, k):
    """S_t = TopK(score, k) ([GLaM] eq. S_t; [GLM45-SE] "keeps the top 8"):
    indices of the k largest scores per token, largest first, exact ties to
    the lower expert index.  A stable sort of -score keeps equal scores in
    index order."""
    sel = _f64(sel)
    order = np.argsort(-sel, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def group_limit(sel, n_group, topk_group):
    """Group-limited selection scores ([GLM45-SE]: the router "optionally
    masks by expert group" before keeping the top k).

    Reading (the note names the step only): experts e in
    [i * M / n_group, (i + 1) * M / n_group) form group i; the group's score
    is the sum of its two largest selection scores (the single score of a
    one-expert group); the topk_group groups with the largest scores stay
    eligible (ties to the lower group index) and the selection score of every
    expert outside them becomes -inf, so the top-k never takes it.  The
    weights still come from the gate values of the chosen experts.
    n_group <= 1 returns the scores unchanged."""
    sel = _f64(sel)
    if n_group is None or n_group <= 1:
        return sel
    T, M = sel.shape
    if M % n_group != 0 or not 1 <= topk_group <= n_group:
        raise ValueError("bad expert grouping")
    size = M // n_group
    per_group = sel.reshape(T, n_group, size)
    best = -np.sort(-per_group, axis=2)[:, :, :min(2, size)]
    group_score = best.sum(axis=2)
    kept = np.argsort(-group_score, axis=1, kind="stable")[:, :topk_group]
    eligible = np.zeros((T, n_group), dtype=bool)
    np.put_along_axis(eligible, kept, True, axis=1)
    return np.where(np.repeat(eligible, size, axis=1), sel, -np.inf)


def topk_weights(idx, logits, g, gate, norm_topk_prob, alpha, eps):
    """Gate weights of the selected experts.

    softmax, normalised ([GLaM] eq. MoE, "normalized gate weight"):
        alpha_j = exp(l_j - l_top) / sum_{i in S} exp(l_i - l_top)
    softmax, not normalised: the full softmax probability of expert j.
    sigmoid_bias ([GLM45-SE] eq. g-bar, then w_i = alpha g-bar_i):
        w_j = alpha * g_j / (sum_{i in S} g_i + eps)   if norm_topk_prob
        w_j = alpha * g_j                              otherwise
    routed_scaling_factor (alpha) multiplies every routed weight."""
    idx = np.asarray(idx)
    if gate == "softmax":
        l = _f64(logits)
        ls = np.take_along_axis(l, idx, axis=1)
        if norm_topk_prob:
            e = np.exp(ls - ls.max(axis=1, keepdims=True))
            w = e / e.sum(axis=1, keepdims=True)
        else:
            full = np.exp(l - l.max(axis=1, keepdims=True))
            full = full / full.sum(axis=1, keepdims=True)
            w = np.take_along_axis(full, idx, axis=1)
        return alpha * w
    if gate == "sigmoid_bias":
        gs = np.take_along_axis(_f64(g), idx, axis=1)
        if norm_topk_prob:
            gs = gs / (gs.sum(axis=1, keepdims=True) + eps)
        return alpha * gs
    raise ValueError(gate)


def route(x, w_r, e_bias, k, gate, norm_topk_prob, alpha, eps, n_group=1, topk_group=1):
    """The whole router: logits, selection (group-limited when n_group > 1),
    weights.  ``sel`` is the unmasked selection score."""
    logits = router_logits(x, w_r)
    sel, g = selection_scores(logits, gate, e_bias)
    idx = topk_select(group_limit(sel, n_group, topk_group), k)
    w = topk_weights(idx, logits, g, gate, norm_topk_prob, alpha, eps)
    return {"logits": logits, "sel": sel, "g": g, "idx": idx, "w": w}


def adopt_topk(gpu_idx, sel, rel=1e-5):
    """Accept a GPU top-k that differs from the oracle's only at near-ties.

    The GPU's choice stands if, for every slot j, the oracle's score of the
    expert the GPU put in slot j lies within ``rel`` (relative) of the j-th
    largest oracle score, and its k indices are distinct and in range.
    Returns (ok, number of tokens whose choice differs, first bad token)."""
    gpu_idx = np.asarray(gpu_idx, dtype=np.int64)
    sel = _f64(sel)
    T, k = gpu_idx.shape
    M = sel.shape[1]
    ref = topk_select(sel, k)
    differ = np.nonzero((gpu_idx != ref).any(axis=1))[0]
    for t in differ:
        g = gpu_idx[t]
        if (g < 0).any() or (g >= M).any() or len(set(g.tolist())) != k:
            return False, len(differ), int(t)
        sg = sel[t, g]
        sr = sel[t, ref[t]]
        band = rel * np.maximum(np.abs(sg), np.abs(sr))
        if (np.abs(sg - sr) > band).any():
            return False, len(differ), int(t)
    return True, len(differ), -1


# ---------------------------------------------------------------------------
# Dispatch
# ---------------------------------------------------------------------------

def permute(idx, w, M):
    """Dispatch order of the (token, slot) pairs.

    [GLM5-SE] GlmMoeDsaExperts.forward: the expert mask one_hot(idx, M + 1)
    permuted to [M + 1, k, T]; ``torch.where(expert_mask[e])`` lists expert
    e's pairs as (slot j, token t) in row-major order, and class M (the
    sentinel) is skipped.  Laying the experts' lists end to end gives a
    stable sort by expert of the pairs taken in (j, t) order.  Returns
      counts[e]       pairs routed to expert e (sentinel pairs not counted)
      offsets[e]      exclusive prefix sum of counts (offsets[M] = pairs kept)
      slot_of[t, j]   position of pair (t, j) in the dispatch order, -1 for
                      a sentinel pair
      row_token[s]    token of the pair at position s
      row_w[s]        its gate weight w[t, j]
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    if ((idx < 0) | (idx > M)).any():
        raise ValueError("expert index outside [0, M]")
    flat = idx.reshape(-1)
    counts = np.bincount(flat[flat < M], minlength=M).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    jmajor = idx.T.reshape(-1)                      # position p = j*T + t
    kept = np.nonzero(jmajor < M)[0]
    order = kept[np.argsort(jmajor[kept], kind="stable")]  # dispatch position -> p
    slot_jmajor = np.full(T * k, -1, dtype=np.int64)
    slot_jmajor[order] = np.arange(order.size)
    slot_of = slot_jmajor.reshape(k, T).T.copy()
    row_token = (order % T).astype(np.int64) if T > 0 else order.astype(np.int64)
    row_w = None
    if w is not None:
        row_w = _f64(w).T.reshape(-1)[order]
    return {"counts": counts, "offsets": offsets, "slot_of": slot_of,
            "row_token": row_token, "row_w": row_w}


def expert_capacity(factor, T, k, M):
    """Pairs an expert may take: ceil(factor * T * k / M).  The pages name no
    capacity rule; this is the plain one, under which a capacity factor of 1
    lets every expert take exactly its even share of the T k pairs."""
    if factor < 0 or M < 1:
        raise ValueError("bad capacity")
    return int(np.ceil(factor * T * k / M - 1e-12)) if T * k > 0 else 0


def capacity_drop(idx, M, capacity):
    """Expert capacity over the dispatch order of ``permute`` (a reading: the
    pages give no rule).  Expert e keeps the first ``capacity`` of its pairs
    in (slot j, then token t) order, so every token's first choice ranks
    before any second choice; each later pair becomes the sentinel M, which
    [GLM5-SE] GlmMoeDsaExperts.forward skips.  Weights are left as they are:
    a dropped pair adds nothing, and the token's other terms keep theirs."""
    idx = np.asarray(idx, dtype=np.int64)
    if capacity < 0:
        raise ValueError("capacity < 0")
    p = permute(idx, None, M)
    out = idx.copy()
    kept = idx < M
    rank = p["slot_of"] - p["offsets"][np.where(kept, idx, 0)]
    out[kept & (rank >= capacity)] = M
    return out


# ---------------------------------------------------------------------------
# Experts
# ---------------------------------------------------------------------------

def expert_ffn(xe, act, w1e, w2e, b1e=None, b2e=None):
    """One expert on a batch of rows xe [n, D].

    gelu_tanh ([GLaM] eq. FFN): W2 sigma(W1 x + b1) + b2, with W1 [H, D],
      W2 [D, H] in the nn.Linear [out, in] layout.
    swiglu ([GLM45-SE] E_sh; [GLM5-SE] GlmMoeDsaExperts.forward): the
      fused stack W1 = gate_up [2I, D]; ``linear(x, gate_up).chunk(2)``
      makes rows 0..I-1 the gate and rows I..2I-1 the up projection;
      E(x) = W_down (SiLU(W_gate x) * W_up x) with W_down = W2 [D, I]."""
    xe = _f64(xe)
    w1e = _f64(w1e)
    w2e = _f64(w2e)
    if act == "gelu_tanh":
        a = xe @ w1e.T
        if b1e is not None:
            a = a + _f64(b1e)[None, :]
        out = gelu_tanh(a) @ w2e.T
        if b2e is not None:
            out = out + _f64(b2e)[None, :]
        return out
    if act == "swiglu":
        I = w1e.shape[0] // 2
        gu = xe @ w1e.T
        h = silu(gu[:, :I]) * gu[:, I:]
        return h @ w2e.T
    raise ValueError(act)


def shared_expert(x, sh_w1, sh_w2):
    """Always-on shared SwiGLU ([GLM45-SE] E_sh; [GLM5-SE] GlmMoeDsaMLP):
    down(SiLU(gate x) * up x) on every token of the pre-routing x, with
    gate/up stored as one [2 I_sh, D] stack (gate rows first)."""
    return expert_ffn(x, "swiglu", sh_w1, sh_w2)


def moe_tokens(x_rows, idx_rows, w_rows, act, get_expert, shared=None, sentinel=None):
    """y_t = sum_{j} w_{t,j} E_{idx[t,j]}(x_t) (+ E_sh(x_t)) for given tokens.

    [GLaM] eq. MoE; [GLM45-SE] eq. y (a sum, no residual inside the layer).
    ``get_expert(e)`` returns (w1e, w2e, b1e, b2e); ``shared`` is
    (sh_w1, sh_w2) or None; pairs whose index equals ``sentinel`` (M) add
    nothing.  Rows that chose expert e are batched into one matmul; each
    row's value is that of its own matrix-vector product."""
    x_rows = _f64(x_rows)
    idx_rows = np.asarray(idx_rows, dtype=np.int64)
    w_rows = _f64(w_rows)
    n, k = idx_rows.shape
    y = np.zeros((n, x_rows.shape[1]), dtype=np.float64)
    for e in np.unique(idx_rows):
        if e < 0:
            raise ValueError("negative expert index")
        if sentinel is not None and e == sentinel:
            continue  # [GLM5-SE]: the sentinel class is skipped
        rr, jj = np.nonzero(idx_rows == e)
        w1e, w2e, b1e, b2e = get_expert(int(e))
        out = expert_ffn(x_rows[rr], act, w1e, w2e, b1e, b2e)
        np.add.at(y, rr, w_rows[rr, jj][:, None] * out)
    if shared is not None:
        y = y + shared_expert(x_rows, shared[0], shared[1])
    return y


def moe_forward(cfg, inp, idx=None, addend=None, w=None):
    """Whole layer: route, dispatch order, experts, combine, shared add.

    ``cfg`` holds T, D, M, k, gate, act, norm_topk_prob, alpha, eps, I_sh;
    ``inp`` holds numpy arrays x, w_r, e_bias, w1, b1, w2, b2, sh_w1, sh_w2
    (w1/w2/b1/b2 indexable by expert).  ``idx`` overrides the selection
    (used when the oracle adopts the GPU's choice at a near-tie); it may hold
    the sentinel M ("no expert", [GLM5-SE] one_hot over M + 1 classes), whose
    pairs add nothing.  ``w`` overrides the gate weights and must be given
    when ``idx`` holds the sentinel (a sentinel has no router score).  With
    ``addend`` the output is the sparse block sum of the "GLaM" note, section
    "Interleaving Dense and Sparse Layers": addend + MoE-FFN(x), addend
    standing for Attention(h)."""
    r = route(inp["x"], inp["w_r"], inp.get("e_bias"), cfg["k"], cfg["gate"],
              cfg["norm_topk_prob"], cfg["alpha"], cfg["eps"], cfg.get("n_group", 1),
              cfg.get("topk_group", 1))
    if idx is not None:
        r["idx"] = np.asarray(idx, dtype=np.int64)
        if w is not None:
            r["w"] = _f64(w)
        elif (r["idx"] == cfg["M"]).any():
            raise ValueError("an index holding the sentinel M needs its gate weights passed as w")
        else:
            r["w"] = topk_weights(r["idx"], r["logits"], r["g"], cfg["gate"],
                                  cfg["norm_topk_prob"], cfg["alpha"], cfg["eps"])
    elif w is not None:
        r["w"] = _f64(w)
    p = permute(r["idx"], r["w"], cfg["M"])

    def get_expert(e):
        b1 = inp.get("b1")
        b2 = inp.get("b2")
        return (inp["w1"][e], inp["w2"][e],
                None if b1 is None else b1[e], None if b2 is None else b2[e])

    shared = None
    if cfg.get("I_sh"):
        shared = (inp["sh_w1"], inp["sh_w2"])
    y = moe_tokens(inp["x"], r["idx"], r["w"], cfg["act"], get_expert, shared, sentinel=cfg["M"])
    if addend is not None:
        y = _f64(addend) + y
    out = dict(r)
    out.update(p)
    out["y"] = y
    return out


def dense_layer(x, act, w1, w2, b1=None, b2=None, addend=None):
    """A dense FFN layer: the "GLaM" note, section "Interleaving Dense and
    Sparse Layers", h^{l+1} = Attention(h^l) + DenseFFN(h^l), with the FFN of
    eq. FFN (GELU form, biases b1, b2); the GLM-4.5 note's dense prefix
    layers, one wide SwiGLU (the same form as an expert, w1 = [gate; up]).
    ``addend`` stands for the other term of the sum (Attention(h), or the
    residual stream); without it the FFN output alone is returned."""
    y = expert_ffn(x, act, w1, w2, b1, b2)
    return y if addend is None else _f64(addend) + y


# ---------------------------------------------------------------------------
# Accounting and comparison
# ---------------------------------------------------------------------------

def param_count(D, M, I, act, I_sh=0, has_bias=False, router=True, e_bias=False):
    """Parameters of one MoE layer ([GLM5-SE] "Exact per-instance
    accounting": gate D*I_sh, up D*I_sh, down I_sh*D for the shared expert;
    the same per routed SwiGLU expert; GELU experts 2*D*H (+ H + D biases);
    the router D*M, plus M correction-bias buffer values)."""
    if act == "swiglu":
        per = 3 * D * I
    else:
        per = 2 * D * I + ((I + D) if has_bias else 0)
    total = M * per + 3 * D * I_sh
    if router:
        total += D * M
    if e_bias:
        total += M
    return total


def error_metrics(y, y_ref):
    """max |y - y_ref| / rms(y_ref) and sum|y - y_ref| / sum|y_ref|."""
    y = _f64(y)
    y_ref = _f64(y_ref)
    d = np.abs(y - y_ref)
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    den = float(np.sum(np.abs(y_ref)))
    return {
        "max_over_rms": float(d.max() / rms) if y_ref.size and rms > 0 else 0.0,
        "mean_rel": float(d.sum() / den) if den > 0 else float(d.sum()),
    }

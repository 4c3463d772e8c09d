"""Plant plausible mistakes in a patched copy of the oracle (on the CPU) and
check that at least one pin fails for each: the pins have teeth."""
import importlib.util
import os

import numpy as np
import pytest

from oracle_pins import ALL_PINS

ORACLE_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                          "oracle", "moe_oracle.py")


def fresh_oracle():
    spec = importlib.util.spec_from_file_location("oracle_mutant", ORACLE_SRC)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def caught(mod):
    for pin in ALL_PINS:
        try:
            pin(mod)
        except AssertionError:
            return pin.__name__
    return None


def m_swap_gate_up(O):
    orig = O.expert_ffn

    def ffn(xe, act, w1e, w2e, b1e=None, b2e=None):
        if act == "swiglu":
            w1e = np.asarray(w1e)
            I = w1e.shape[0] // 2
            w1e = np.concatenate([w1e[I:], w1e[:I]])
        return orig(xe, act, w1e, w2e, b1e, b2e)
    O.expert_ffn = ffn


def m_drop_b2(O):
    orig = O.expert_ffn
    O.expert_ffn = lambda xe, act, w1e, w2e, b1e=None, b2e=None: orig(xe, act, w1e, w2e, b1e, None)


def m_bias_in_weights(O):
    orig = O.selection_scores
    O.selection_scores = lambda logits, gate, e_bias=None: (
        orig(logits, gate, e_bias)[0], orig(logits, gate, e_bias)[0])


def _grouped(O, group_score, masked_value=-np.inf, tie_high=False):
    def group_limit(sel, n_group, topk_group):
        sel = np.asarray(sel, np.float64)
        if n_group <= 1:
            return sel
        T, M = sel.shape
        size = M // n_group
        gs = group_score(sel.reshape(T, n_group, size))
        if tie_high:
            order = n_group - 1 - np.argsort(-gs[:, ::-1], axis=1, kind="stable")
        else:
            order = np.argsort(-gs, axis=1, kind="stable")
        keep = np.zeros((T, n_group), bool)
        np.put_along_axis(keep, order[:, :topk_group], True, axis=1)
        return np.where(np.repeat(keep, size, axis=1), sel, masked_value)
    O.group_limit = group_limit


def _top2_sum(g):
    return (-np.sort(-g, axis=2))[:, :, :2].sum(axis=2)


def m_group_score_max(O):
    _grouped(O, lambda g: g.max(axis=2))


def m_group_score_all(O):
    _grouped(O, lambda g: g.sum(axis=2))


def m_group_mask_zero(O):
    _grouped(O, _top2_sum, masked_value=0.0)


def m_group_tie_high(O):
    _grouped(O, _top2_sum, tie_high=True)


def m_tie_to_higher_index(O):
    def topk(sel, k):
        sel = np.asarray(sel, np.float64)
        M = sel.shape[1]
        rev = np.argsort(-sel[:, ::-1], axis=1, kind="stable")
        return (M - 1 - rev)[:, :k].astype(np.int64)
    O.topk_select = topk


def m_no_renorm(O):
    orig = O.topk_weights
    O.topk_weights = lambda idx, l, g, gate, norm, a, eps: orig(idx, l, g, gate, 0, a, eps)


def m_no_alpha(O):
    orig = O.topk_weights
    O.topk_weights = lambda idx, l, g, gate, norm, a, eps: orig(idx, l, g, gate, norm, 1.0, eps)


def m_token_major_dispatch(O):
    def permute(idx, w, M):
        idx = np.asarray(idx, np.int64)
        T, k = idx.shape
        order = np.argsort(idx.reshape(-1), kind="stable")  # (t, j) order: wrong
        slot = np.empty(T * k, np.int64)
        slot[order] = np.arange(T * k)
        counts = np.bincount(idx.reshape(-1), minlength=M)
        return {"counts": counts, "offsets": np.concatenate([[0], np.cumsum(counts)]),
                "slot_of": slot.reshape(T, k), "row_token": order // k,
                "row_w": np.asarray(w, np.float64).reshape(-1)[order]}
    O.permute = permute


def m_gelu_erf(O):
    from math import erf
    O.gelu_tanh = lambda v: np.vectorize(lambda a: 0.5 * a * (1 + erf(a / np.sqrt(2))))(np.asarray(v, np.float64))


def m_shared_missing(O):
    O.shared_expert = lambda x, a, b: np.zeros((np.asarray(x).shape[0], np.asarray(b).shape[0]))


def m_transposed_router(O):
    O.router_logits = lambda x, w_r: np.asarray(x, np.float64) @ np.asarray(w_r, np.float64)[::-1, :]


def m_wrong_param_count(O):
    orig = O.param_count
    O.param_count = lambda D, M, I, act, I_sh=0, **kw: orig(D, M, I, act, I_sh=I_sh, **kw) - (2 * D * I_sh)


def m_dense_drops_addend(O):
    orig = O.dense_layer
    O.dense_layer = lambda x, act, w1, w2, b1=None, b2=None, addend=None: orig(x, act, w1, w2, b1, b2)


def m_block_drops_addend(O):
    orig = O.moe_forward
    O.moe_forward = lambda cfg, inp, idx=None, addend=None, w=None: orig(cfg, inp, idx, w=w)


def m_dense_no_b2(O):
    orig = O.dense_layer
    O.dense_layer = lambda x, act, w1, w2, b1=None, b2=None, addend=None: orig(x, act, w1, w2, b1, None,
                                                                                addend)


def m_capacity_token_major(O):
    def drop(idx, M, capacity):
        idx = np.asarray(idx, np.int64)
        out = idx.copy()
        seen = np.zeros(M, np.int64)
        for t in range(idx.shape[0]):          # token first: a later token's first choice loses
            for j in range(idx.shape[1]):
                e = idx[t, j]
                if e < M:
                    if seen[e] >= capacity:
                        out[t, j] = M
                    seen[e] += 1
        return out
    O.capacity_drop = drop


def m_capacity_off_by_one(O):
    orig = O.capacity_drop
    O.capacity_drop = lambda idx, M, capacity: orig(idx, M, capacity + 1)


MUTANTS = [m_swap_gate_up, m_drop_b2, m_bias_in_weights, m_tie_to_higher_index,
           m_no_renorm, m_no_alpha, m_token_major_dispatch, m_gelu_erf,
           m_shared_missing, m_transposed_router, m_wrong_param_count, m_group_score_max,
           m_group_score_all, m_group_mask_zero, m_group_tie_high, m_dense_drops_addend, m_dense_no_b2,
           m_block_drops_addend, m_capacity_token_major, m_capacity_off_by_one]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda f: f.__name__)
def test_mutant_is_caught(mutant):
    O = fresh_oracle()
    assert caught(O) is None, "unpatched oracle must pass every pin"
    mutant(O)
    assert caught(O) is not None, f"no pin caught {mutant.__name__}"

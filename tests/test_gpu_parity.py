"""Parity of the CUDA path (called through the C ABI) with the CPU oracle on
identical seeded inputs, stage by stage and for the whole layer."""
import numpy as np
import pytest
import torch

import moe_synth as ms
import oracle
from gpu_common import (check_permutation, check_routing, check_y, gpu_inputs, np64, oracle_route,
                        oracle_y, sample_tokens, tile_tokens)

pytestmark = pytest.mark.gpu

SMALL = ["glam_tiny_f32", "glam_small_bf16", "glm_small_bf16", "glm_medium_bf16", "glm_small_f32",
         "glam_nonorm_f32", "glm_grouped_bf16", "glm_grouped_f32"]
FULL = ["glam_prefill_bf16", "glm45_decode_bf16", "glm45_prefill_bf16", "glm5_skewed_prefill_bf16"]


@pytest.fixture(scope="module")
def B():
    import sparse_mixture_experts_logits_b200 as B
    return B


def run_forward(B, cfg, inp):
    layer = B.MoELayer(cfg, inp)
    y = layer.forward(inp["x"])
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    views = {n: layer.view(n).cpu().numpy() for n in
             ("topk_idx", "topk_w", "counts", "offsets", "slot_of", "row_token", "row_w")}
    return layer, y, views


def check_layer(B, cfg, all_tokens=True):
    """all_tokens: True compares y on every token; "tiles" on the tokens of
    the first, last and one middle row of every token tile of the expert and
    shared GEMMs (so every tile is compared at full K); False on a sample."""
    inp = gpu_inputs(cfg)
    layer, y, v = run_forward(B, cfg, inp)
    r = oracle_route(cfg, inp)
    w_ref, ndiff = check_routing(cfg, r, v["topk_idx"], v["topk_w"])
    p = check_permutation(cfg, v["topk_idx"], v["topk_w"], v)
    if all_tokens is True:
        tokens = np.arange(cfg["T"])
    elif all_tokens == "tiles":
        tokens = tile_tokens(cfg, p["counts"], p["row_token"], p["offsets"])
    else:
        tokens = sample_tokens(cfg, p["counts"], p["row_token"], p["offsets"])
    y_ref = oracle_y(cfg, inp, tokens, v["topk_idx"], w_ref)
    m = check_y(cfg, np64(y[torch.as_tensor(tokens, device=y.device)]), y_ref)
    return layer, inp, y, v, m, ndiff


@pytest.mark.parametrize("name", SMALL)
def test_small_layer_all_tokens(B, name):
    check_layer(B, ms.get_config(name), all_tokens=True)


# GLaM prefill and decode: y on every token; the GLM prefill layers: y on
# the tokens of every token tile of every expert segment (first, last and a
# middle row), which covers each tile of both expert GEMMs at full K.
FULL_TOKENS = {"glam_prefill_bf16": True, "glm45_decode_bf16": True, "glm45_prefill_bf16": "tiles",
               "glm5_skewed_prefill_bf16": "tiles"}


@pytest.mark.parametrize("name", FULL)
def test_full_size_layer(B, name):
    """Full-size workloads in the benchmark's launch configuration: routing
    and dispatch checked on every token, y on every token or on every token
    tile of the expert GEMMs, at the literal bound."""
    _, _, _, _, m, _ = check_layer(B, ms.get_config(name), all_tokens=FULL_TOKENS[name])
    print(name, m)


def test_group_limited_full_size(B):
    """The GLM-5 skewed prefill layer with the router limited to the 4 best
    of 8 expert groups (32 experts each), y on every token tile."""
    check_layer(B, ms.get_config("glm5_skewed_prefill_bf16", n_group=8, topk_group=4), all_tokens="tiles")


@pytest.mark.parametrize("name,over", [
    ("glm_small_bf16", dict(T=1)),
    ("glm_small_bf16", dict(T=15)),                      # few rows: the shared expert on the side stream
    ("glm_small_bf16", dict(T=128)),
    ("glm_small_bf16", dict(T=129)),
    ("glm_small_bf16", dict(T=64, I_sh=208)),            # a shared gate/up width not a multiple of 32
    ("glm_medium_bf16", dict(T=40)),                     # few tokens, I_sh = 320, D = 512
    ("glm_small_bf16", dict(k=1)),
    ("glm_small_bf16", dict(M=4, k=4)),
    ("glam_small_bf16", dict(M=1, k=1)),
    ("glam_small_bf16", dict(T=2000, norm_topk_prob=0)),
    ("glm_small_bf16", dict(I_sh=0)),
    ("glm_small_bf16", dict(e_bias=("const", 0.0), alpha=1.0)),
    ("glm_medium_bf16", dict(e_bias=("zipf", 1.1, 1.0))),  # literal beta = 1: most experts empty
    ("glam_tiny_f32", dict(T=1)),
    ("glam_small_bf16", dict(T=5)),                      # GELU experts on the few-rows (tokens-on-M) path
    ("glm_small_bf16", dict(n_group=16, topk_group=4)),  # one expert per group
    ("glm_small_bf16", dict(n_group=4, topk_group=4)),   # every group kept
    ("glm_small_bf16", dict(n_group=4, topk_group=1)),   # k = the whole kept group
    ("glam_small_bf16", dict(n_group=2, topk_group=1)),  # softmax router, groups of 4
    ("glm_small_bf16", dict(M=1024, k=32)),              # the largest M and k the library takes
    ("glm_small_f32", dict(M=1024, k=32, T=40)),         # the same on the fp32 path
    ("glam_small_bf16", dict(M=64, k=32)),               # softmax router, k = 32
    ("glam_small_bf16", dict(T=40000)),                  # many dispatch chunks, ragged tail
    ("glm_small_bf16", dict(M=1024, k=32, n_group=32, topk_group=4)),  # 32 groups of 32
])
def test_edge_cases(B, name, over):
    check_layer(B, ms.get_config(name, **over), all_tokens=True)


def test_all_tokens_to_few_experts(B):
    """A correction bias that sends every token to the same k experts: k
    segments of T rows each (several m-tiles), every other expert empty."""
    cfg = ms.get_config("glm_small_bf16", T=700)
    inp = gpu_inputs(cfg)
    bias = torch.zeros(cfg["M"], device="cuda")
    bias[[3, 5, 11, 12]] = 10.0
    inp["e_bias"] = bias
    layer, y, v = run_forward(B, cfg, inp)
    assert sorted(np.nonzero(v["counts"])[0].tolist()) == [3, 5, 11, 12]
    r = oracle_route(cfg, inp)
    w_ref, _ = check_routing(cfg, r, v["topk_idx"], v["topk_w"])
    check_permutation(cfg, v["topk_idx"], v["topk_w"], v)
    y_ref = oracle_y(cfg, inp, np.arange(cfg["T"]), v["topk_idx"], w_ref)
    check_y(cfg, np64(y), y_ref)


def test_deterministic(B):
    cfg = ms.get_config("glm_medium_bf16")
    inp = gpu_inputs(cfg)
    layer = B.MoELayer(cfg, inp)
    y1 = layer.forward(inp["x"]).clone()
    y2 = layer.forward(inp["x"])
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_stage_entry_points_match_forward(B):
    """moe_route_topk, moe_permute, moe_expert_ffn, moe_shared_expert and
    moe_combine called one by one give the forward's intermediates."""
    cfg = ms.get_config("glm_small_bf16")
    inp = gpu_inputs(cfg)
    layer, y, v = run_forward(B, cfg, inp)
    d = layer.desc
    T, D, M, k = cfg["T"], cfg["D"], cfg["M"], cfg["k"]
    dev = "cuda"
    s = torch.cuda.current_stream().cuda_stream

    def ws(nbytes):
        return torch.zeros(nbytes + 256, dtype=torch.uint8, device=dev)

    idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    w = torch.empty(T, k, dtype=torch.float32, device=dev)
    wr = ws(B.moe_route_workspace_size(T, D, M, d.dtype))
    B.moe_route_topk(inp["x"].data_ptr(), inp["w_r"].data_ptr(), inp["e_bias"].data_ptr(), T, D, M, k,
                     d.dtype, d.gate, d.norm_topk_prob, d.routed_scaling_factor, d.eps, d.n_group,
                     d.topk_group, idx.data_ptr(),
                     w.data_ptr(), wr.data_ptr(), wr.numel(), s)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), v["topk_idx"])
    assert np.array_equal(w.cpu().numpy(), v["topk_w"])

    counts = torch.empty(M, dtype=torch.int32, device=dev)
    offsets = torch.empty(M + 1, dtype=torch.int32, device=dev)
    slot_of = torch.empty(T, k, dtype=torch.int32, device=dev)
    row_token = torch.empty(T * k, dtype=torch.int32, device=dev)
    row_w = torch.empty(T * k, dtype=torch.float32, device=dev)
    wp = ws(B.moe_permute_workspace_size(T, k, M))
    B.moe_permute(idx.data_ptr(), w.data_ptr(), T, k, M, counts.data_ptr(), offsets.data_ptr(),
                  slot_of.data_ptr(), row_token.data_ptr(), row_w.data_ptr(), wp.data_ptr(), wp.numel(), s)
    torch.cuda.synchronize()
    for name, t in [("counts", counts), ("offsets", offsets), ("slot_of", slot_of),
                    ("row_token", row_token), ("row_w", row_w)]:
        assert np.array_equal(t.cpu().numpy(), v[name]), name

    out_perm = torch.empty(T * k, D, dtype=torch.float32, device=dev)
    wf = ws(B.moe_expert_ffn_workspace_size(d))
    B.moe_expert_ffn(d, layer.weights, inp["x"].data_ptr(), offsets.data_ptr(), row_token.data_ptr(),
                     row_w.data_ptr(), out_perm.data_ptr(), wf.data_ptr(), wf.numel(), s)
    torch.cuda.synchronize()
    assert torch.equal(out_perm.view(torch.int32), layer.view("out_perm").view(torch.int32))
    # each dispatched row against the oracle: row_w[s] * E_e(x[row_token[s]])
    offs = v["offsets"]
    xs = np64(inp["x"])
    for e in range(M):
        rows = np.arange(offs[e], offs[e + 1])
        if rows.size == 0:
            continue
        ref = oracle.expert_ffn(xs[v["row_token"][rows]], cfg["act"], np64(inp["w1"][e]),
                                np64(inp["w2"][e])) * v["row_w"][rows][:, None]
        m = oracle.error_metrics(np64(out_perm[torch.as_tensor(rows, device=dev)]), ref)
        assert m["mean_rel"] < 5e-3 and m["max_over_rms"] < 2e-2, (e, m)

    y_sh = torch.empty(T, D, dtype=torch.bfloat16, device=dev)
    wsh = ws(B.moe_shared_expert_workspace_size(d))
    B.moe_shared_expert(d, layer.weights, inp["x"].data_ptr(), y_sh.data_ptr(), wsh.data_ptr(),
                        wsh.numel(), s)
    y_c = torch.empty(T, D, dtype=torch.bfloat16, device=dev)
    B.moe_combine(d, out_perm.data_ptr(), slot_of.data_ptr(), y_sh.data_ptr(), None, y_c.data_ptr(), s)
    torch.cuda.synchronize()
    sh_ref = oracle.shared_expert(xs, np64(inp["sh_w1"]), np64(inp["sh_w2"]))
    m = oracle.error_metrics(np64(y_sh), sh_ref)
    assert m["mean_rel"] < 5e-3 and m["max_over_rms"] < 2e-2, m
    # unfused combine (shared output rounded to bf16, then added) against the oracle
    w_ref = oracle.topk_weights(v["topk_idx"], *[oracle_route(cfg, inp)[n] for n in ("logits", "g")],
                                cfg["gate"], cfg["norm_topk_prob"], cfg["alpha"], cfg["eps"])
    check_y(dict(cfg, named=False), np64(y_c), oracle_y(cfg, inp, np.arange(T), v["topk_idx"], w_ref))


def test_bad_expert_index_is_reported_not_faulted(B):
    T, k, M = 100, 2, 8
    dev = "cuda"
    idx = torch.randint(0, M, (T, k), dtype=torch.int32, device=dev)
    idx[17, 1] = M + 5
    idx[3, 0] = -2
    w = torch.rand(T, k, device=dev)
    outs = [torch.empty(n, dtype=dt, device=dev) for n, dt in
            [(M, torch.int32), (M + 1, torch.int32), (T * k, torch.int32), (T * k, torch.int32),
             (T * k, torch.float32)]]
    nbytes = B.moe_permute_workspace_size(T, k, M)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    B.moe_permute(idx.data_ptr(), w.data_ptr(), T, k, M, *[o.data_ptr() for o in outs], ws.data_ptr(),
                  nbytes, s)
    assert B.moe_device_status(ws.data_ptr(), s) == B.DEVERR_BAD_EXPERT_INDEX
    assert B.moe_device_status(ws.data_ptr(), s) == 0  # read clears it
    assert int(outs[0].sum()) == T * k - 2


@pytest.mark.parametrize("name,frac", [("glm_small_bf16", 0.25), ("glam_small_bf16", 0.4),
                                       ("glm_small_f32", 0.3), ("glm_medium_bf16", 0.6)])
def test_sentinel_pairs_are_dispatched_nowhere(B, name, frac):
    """Expert index M marks a dropped pair (the GLM-5 page's expert mask over
    M + 1 classes, class M skipped): moe_permute dispatches it nowhere
    (slot_of = -1, not counted), moe_combine adds nothing for it."""
    cfg = ms.get_config(name)
    inp = gpu_inputs(cfg)
    T, D, M, k = cfg["T"], cfg["D"], cfg["M"], cfg["k"]
    r = oracle_route(cfg, inp)
    idx = r["idx"].copy()
    drop = np.random.default_rng(3).random(idx.shape) < frac
    idx[drop] = M
    w32 = r["w"].astype(np.float32)
    dev = "cuda"
    s = torch.cuda.current_stream().cuda_stream
    idx_d = torch.as_tensor(idx, dtype=torch.int32, device=dev)
    w_d = torch.as_tensor(w32, device=dev)
    counts = torch.empty(M, dtype=torch.int32, device=dev)
    offsets = torch.empty(M + 1, dtype=torch.int32, device=dev)
    slot_of = torch.empty(T, k, dtype=torch.int32, device=dev)
    row_token = torch.empty(T * k, dtype=torch.int32, device=dev)
    row_w = torch.empty(T * k, dtype=torch.float32, device=dev)
    nbytes = B.moe_permute_workspace_size(T, k, M)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    B.moe_permute(idx_d.data_ptr(), w_d.data_ptr(), T, k, M, counts.data_ptr(), offsets.data_ptr(),
                  slot_of.data_ptr(), row_token.data_ptr(), row_w.data_ptr(), ws.data_ptr(), nbytes, s)
    assert B.moe_device_status(ws.data_ptr(), s) == 0
    p = oracle.permute(idx, w32.astype(np.float64), M)
    kept = int(p["offsets"][M])
    assert np.array_equal(counts.cpu().numpy(), p["counts"])
    assert np.array_equal(offsets.cpu().numpy(), p["offsets"])
    assert np.array_equal(slot_of.cpu().numpy(), p["slot_of"])
    assert np.array_equal(row_token.cpu().numpy()[:kept], p["row_token"])
    assert np.array_equal(row_w.cpu().numpy()[:kept].astype(np.float64), p["row_w"])

    d = B.desc_from_config(cfg)
    weights = B.weights_from_tensors(inp)
    out_perm = torch.empty(T * k, D, dtype=torch.float32, device=dev)
    wf = torch.zeros(B.moe_expert_ffn_workspace_size(d) + 256, dtype=torch.uint8, device=dev)
    B.moe_expert_ffn(d, weights, inp["x"].data_ptr(), offsets.data_ptr(), row_token.data_ptr(),
                     row_w.data_ptr(), out_perm.data_ptr(), wf.data_ptr(), wf.numel(), s)
    shared_out = None
    if cfg.get("I_sh"):
        shared_out = torch.empty_like(inp["x"])
        wsh = torch.zeros(B.moe_shared_expert_workspace_size(d) + 256, dtype=torch.uint8, device=dev)
        B.moe_shared_expert(d, weights, inp["x"].data_ptr(), shared_out.data_ptr(), wsh.data_ptr(),
                            wsh.numel(), s)
    y = torch.empty_like(inp["x"])
    B.moe_combine(d, out_perm.data_ptr(), slot_of.data_ptr(),
                  None if shared_out is None else shared_out.data_ptr(), None, y.data_ptr(), s)
    torch.cuda.synchronize()
    shared = (np64(inp["sh_w1"]), np64(inp["sh_w2"])) if cfg.get("I_sh") else None
    from gpu_common import HostExperts
    y_ref = oracle.moe_tokens(np64(inp["x"]), idx, w32.astype(np.float64), cfg["act"], HostExperts(inp),
                              shared, sentinel=M)
    check_y(dict(cfg, named=False), np64(y), y_ref)


def test_bad_row_token_is_reported_not_faulted(B):
    """A dispatch row whose token index is outside [0, T) is read as zeros
    and reported through the status flag; the other rows are unaffected."""
    cfg = ms.get_config("glm_small_bf16")
    inp = gpu_inputs(cfg)
    layer, y, v = run_forward(B, cfg, inp)
    d = layer.desc
    T, D, k = cfg["T"], cfg["D"], cfg["k"]
    dev = "cuda"
    s = torch.cuda.current_stream().cuda_stream
    offsets = torch.as_tensor(v["offsets"], device=dev)
    row_token = torch.as_tensor(v["row_token"], device=dev).clone()
    row_w = torch.as_tensor(v["row_w"], device=dev)
    bad = [5, T * k // 2]
    row_token[bad[0]] = T + 3
    row_token[bad[1]] = -1
    out_perm = torch.empty(T * k, D, dtype=torch.float32, device=dev)
    wf = torch.zeros(B.moe_expert_ffn_workspace_size(d) + 256, dtype=torch.uint8, device=dev)
    B.moe_expert_ffn(d, layer.weights, inp["x"].data_ptr(), offsets.data_ptr(), row_token.data_ptr(),
                     row_w.data_ptr(), out_perm.data_ptr(), wf.data_ptr(), wf.numel(), s)
    assert B.moe_device_status(wf.data_ptr(), s) == B.DEVERR_BAD_ROW_TOKEN
    ref = layer.view("out_perm")
    keep = torch.ones(T * k, dtype=torch.bool, device=dev)
    keep[bad] = False
    assert torch.equal(out_perm[keep].view(torch.int32), ref[keep].view(torch.int32))
    assert torch.isfinite(out_perm[bad]).all()


def test_zero_routed_scale_leaves_the_shared_expert(B):
    """With routed_scaling_factor 0 every routed term is an exact zero, so y is
    the shared expert's output alone ("Shared Expert" GLM-4.5 note: E_sh reads
    the pre-routing x), bit for bit the standalone moe_shared_expert."""
    cfg = ms.get_config("glm_small_bf16", alpha=0.0)
    inp = gpu_inputs(cfg)
    layer, y, _ = run_forward(B, cfg, inp)
    d = layer.desc
    y_sh = torch.empty_like(inp["x"])
    wsh = torch.zeros(B.moe_shared_expert_workspace_size(d) + 256, dtype=torch.uint8, device="cuda")
    B.moe_shared_expert(d, layer.weights, inp["x"].data_ptr(), y_sh.data_ptr(), wsh.data_ptr(), wsh.numel(),
                        torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_sh.view(torch.int16))


@pytest.mark.parametrize("seed", range(8))
def test_random_shapes(B, seed):
    """Seeded random layers inside the library's limits: widths, expert
    counts, k, router and expert kinds, token counts with ragged tails."""
    rng = np.random.default_rng(100 + seed)
    swiglu = bool(rng.integers(0, 2))
    M = int(rng.choice([2, 5, 8, 12, 16, 24, 40, 64]))
    k = int(rng.integers(1, min(M, 8) + 1))
    over = dict(T=int(rng.integers(1, 700)), D=int(16 * rng.integers(2, 24)),
                I=int(16 * rng.integers(1, 24)), M=M, k=k, seed=seed)
    name = "glm_small_bf16" if swiglu else "glam_small_bf16"
    if swiglu:
        over["I_sh"] = int(16 * rng.integers(0, 12))
    check_layer(B, ms.get_config(name, **over), all_tokens=True)

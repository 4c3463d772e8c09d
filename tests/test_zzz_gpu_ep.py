"""The expert-parallel exchange on one GPU.

moe_ep_pack and moe_ep_unpack are index work: they are compared bit for bit
with their definitions (the header's statement, restated here on the host),
on dispatch orders from the oracle's permutation and on synthetic arrival
layouts of 1 to 4 source ranks.  The whole expert-parallel layer
(sparse_mixture_experts_logits_b200.ep) then runs at world = 1, every expert
local and each exchange a copy, and its y is compared with the oracle's
layer with the pairs past an expert's capacity dropped.  Collected after the
forward suites (test_zzz_*)."""
import numpy as np
import pytest
import torch

import moe_synth as ms
import oracle
from gpu_common import HostExperts, check_routing, check_y, gpu_inputs, np64, oracle_route

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    import sparse_mixture_experts_logits_b200 as B
    return B


def _pack_reference(x, p, M, cap):
    """moe_ep_pack as the header states it (host)."""
    off, rt, rw = p["offsets"], p["row_token"], p["row_w"]
    D = x.shape[1]
    x_pad = np.zeros((M * cap, D), dtype=x.dtype)
    w_pad = np.zeros(M * cap, dtype=np.float32)
    kept = np.zeros(M, dtype=np.int32)
    for e in range(M):
        n = int(off[e + 1] - off[e])
        kept[e] = min(n, cap)
        for i in range(kept[e]):
            x_pad[e * cap + i] = x[rt[off[e] + i]]
            w_pad[e * cap + i] = rw[off[e] + i]
    so = p["slot_of"].reshape(-1)
    slot_pad = np.full(so.shape, -1, dtype=np.int32)
    for q, s in enumerate(so):
        if s >= 0:
            e = int(np.searchsorted(off, s, side="right") - 1)
            if s - off[e] < cap:
                slot_pad[q] = e * cap + (s - off[e])
    return x_pad, w_pad, slot_pad, kept


@pytest.mark.parametrize("T,k,M,cap,dtype", [(300, 4, 16, 300, "bf16"), (300, 4, 16, 75, "bf16"),
                                             (77, 3, 12, 5, "f32"), (64, 2, 8, 0, "bf16"),
                                             (1, 1, 4, 1, "f32"), (0, 2, 8, 3, "bf16")])
def test_ep_pack_matches_definition(B, T, k, M, cap, dtype):
    g = np.random.default_rng(T * 7 + cap)
    D = 48
    idx = np.stack([g.choice(M, size=k, replace=False) for _ in range(T)]).reshape(T, k) if T else \
        np.zeros((0, k), dtype=np.int64)
    w = g.random((T, k))
    p = oracle.permute(idx, w, M)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = torch.randn(max(T, 1), D, dtype=torch.float32).to(tdt)[:T].contiguous().cuda()
    dev = {name: torch.as_tensor(np.asarray(p[name]), dtype=torch.int32 if name != "row_w" else torch.float32)
           .reshape(-1).cuda() for name in ("offsets", "row_token", "row_w", "slot_of")}
    x_pad = torch.full((M * cap, D), 7.0, dtype=tdt, device="cuda")
    w_pad = torch.full((M * cap,), 7.0, device="cuda")
    slot_pad = torch.full((T * k,), 7, dtype=torch.int32, device="cuda")
    kept = torch.full((M,), 7, dtype=torch.int32, device="cuda")
    status = torch.full((1,), 9, dtype=torch.int32, device="cuda")
    B.moe_ep_pack(x.data_ptr() if T else None, dev["offsets"].data_ptr(), dev["row_token"].data_ptr(),
                  dev["row_w"].data_ptr(), dev["slot_of"].data_ptr(), T, k, M, D,
                  B.DTYPE_BF16 if dtype == "bf16" else B.DTYPE_F32, cap, x_pad.data_ptr() if cap else None,
                  w_pad.data_ptr() if cap else None, slot_pad.data_ptr() if T else None, kept.data_ptr(),
                  status.data_ptr(), None)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    xr, wr, sr, kr = _pack_reference(x.cpu().float().numpy() if T else np.zeros((0, D), np.float32),
                                     {n: np.asarray(p[n]) for n in ("offsets", "row_token", "row_w", "slot_of")},
                                     M, cap)
    assert np.array_equal(kept.cpu().numpy(), kr)
    assert np.array_equal(slot_pad.cpu().numpy(), sr)
    assert np.array_equal(w_pad.cpu().numpy(), wr)
    assert np.array_equal(x_pad.cpu().float().numpy(), xr)


def _unpack_reference(recv_kept, w_recv, world, E, cap):
    """moe_ep_unpack as the header states it (host)."""
    kept = np.clip(recv_kept.reshape(world, E), 0, cap)
    offsets = np.zeros(E + 1, dtype=np.int32)
    row_token, row_w = [], []
    slot_of = np.full(world * E * cap, -1, dtype=np.int32)
    for e in range(E):
        offsets[e] = len(row_token)
        for q in range(world):
            for i in range(kept[q, e]):
                r = (q * E + e) * cap + i
                slot_of[r] = len(row_token)
                row_token.append(r)
                row_w.append(w_recv[r])
    offsets[E] = len(row_token)
    return offsets, np.asarray(row_token, np.int32), np.asarray(row_w, np.float32), slot_of


@pytest.mark.parametrize("world,E,cap,bad", [(1, 8, 40, False), (2, 4, 17, False), (4, 3, 9, False),
                                             (4, 64, 33, False), (2, 5, 6, True), (3, 2, 0, False)])
def test_ep_unpack_matches_definition(B, world, E, cap, bad):
    g = np.random.default_rng(world * 100 + E)
    recv_kept = g.integers(0, cap + 1, size=world * E).astype(np.int32)
    if bad:
        recv_kept[1], recv_kept[3] = cap + 4, -2       # clamped, and reported
    w_recv = g.random(world * E * cap).astype(np.float32)
    R = world * E * cap
    d_kept = torch.as_tensor(recv_kept).cuda()
    d_w = torch.as_tensor(w_recv).cuda()
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    row_token = torch.full((max(R, 1),), -7, dtype=torch.int32, device="cuda")
    row_w = torch.full((max(R, 1),), -7.0, device="cuda")
    slot_of = torch.full((max(R, 1),), -7, dtype=torch.int32, device="cuda")
    status = torch.full((1,), 9, dtype=torch.int32, device="cuda")
    B.moe_ep_unpack(d_kept.data_ptr(), d_w.data_ptr() if R else None, world, E, cap, offsets.data_ptr(),
                    row_token.data_ptr() if R else None, row_w.data_ptr() if R else None,
                    slot_of.data_ptr() if R else None, status.data_ptr(), None)
    torch.cuda.synchronize()
    assert int(status.item()) == (B.DEVERR_BAD_COUNT if bad else 0)
    o, rt, rw, so = _unpack_reference(recv_kept, w_recv, world, E, cap)
    n = int(o[E])
    assert np.array_equal(offsets.cpu().numpy(), o)
    assert np.array_equal(row_token.cpu().numpy()[:n], rt)
    assert np.array_equal(row_w.cpu().numpy()[:n], rw)
    if R:
        assert np.array_equal(slot_of.cpu().numpy()[:R], so)


def ep_layer(cfg, inp, factor):
    from sparse_mixture_experts_logits_b200 import ep
    return ep.ExpertParallelMoE(cfg, ep.local_expert_tensors(inp, 0, 1), rank=0, world=1,
                                capacity_factor=factor)


@pytest.mark.parametrize("name,factor", [("glam_small_bf16", None), ("glam_tiny_f32", None),
                                         ("glm_small_bf16", None), ("glm_grouped_bf16", None),
                                         ("glm_small_bf16", 1.0), ("glam_small_bf16", 0.5),
                                         ("glm_small_f32", 0.75)])
def test_expert_parallel_one_rank_matches_oracle(B, name, factor):
    from sparse_mixture_experts_logits_b200 import ep
    cfg = ms.get_config(name)
    T, k, M = cfg["T"], cfg["k"], cfg["M"]
    inp = gpu_inputs(cfg)
    layer = ep_layer(cfg, inp, factor)
    y = layer.forward(inp["x"])
    y2 = layer.forward(inp["x"]).clone()               # the buffers are reused: same result
    torch.cuda.synchronize()
    assert layer.status.tolist() == [0, 0]
    b = layer.buffers(T, inp["x"].dtype)
    idx, tw = b["idx"].cpu().numpy(), b["tw"].cpu().numpy()
    w_ref, _ = check_routing(cfg, oracle_route(cfg, inp), idx, tw)
    cap = ep.capacity(T, k, M, factor)
    kept_idx = oracle.capacity_drop(idx, M, cap)
    if factor is None:
        assert (kept_idx < M).all()
    elif factor < 1:
        assert (kept_idx == M).any()                  # the capacity bites
    counts = np.bincount(idx.reshape(-1), minlength=M)
    assert np.array_equal(b["kept"].cpu().numpy(), np.minimum(counts, cap))
    shared = (np64(inp["sh_w1"]), np64(inp["sh_w2"])) if cfg.get("I_sh") else None
    y_ref = oracle.moe_tokens(np64(inp["x"]), kept_idx, w_ref, cfg["act"], HostExperts(inp), shared, sentinel=M)
    check_y(dict(cfg, named=False), np64(y), y_ref)
    view = torch.int16 if y.dtype == torch.bfloat16 else torch.int32
    assert torch.equal(y.view(view), y2.view(view))


@pytest.mark.parametrize("name", ["glam_small_bf16", "glam_tiny_f32"])
def test_expert_parallel_one_rank_equals_forward_without_drops(B, name):
    """No shared expert and no drops: the same rows go through the same
    kernels in the same per-expert order, so y equals moe_forward's bit for
    bit."""
    cfg = ms.get_config(name)
    inp = gpu_inputs(cfg)
    y_ep = ep_layer(cfg, inp, None).forward(inp["x"])
    y = B.MoELayer(cfg, inp).forward(inp["x"])
    torch.cuda.synchronize()
    view = torch.int16 if y.dtype == torch.bfloat16 else torch.int32
    assert torch.equal(y_ep.view(view), y.view(view))

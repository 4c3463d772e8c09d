"""Expert capacity on the GPU (moe_capacity_drop) against the oracle's
capacity_drop, then the layer over the kept pairs (moe_permute again,
experts, combine with the sentinel skipped) against the oracle.  Collected
after the forward suites (test_zzz_*)."""
import numpy as np
import pytest
import torch

import moe_synth as ms
import oracle
from gpu_common import HostExperts, check_y, gpu_inputs, np64, oracle_route

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    import sparse_mixture_experts_logits_b200 as B
    return B


def _permute(B, idx_d, w_d, T, k, M, s):
    dev = idx_d.device
    out = {"counts": torch.empty(M, dtype=torch.int32, device=dev),
           "offsets": torch.empty(M + 1, dtype=torch.int32, device=dev),
           "slot_of": torch.empty(T, k, dtype=torch.int32, device=dev),
           "row_token": torch.empty(T * k, dtype=torch.int32, device=dev),
           "row_w": torch.empty(T * k, dtype=torch.float32, device=dev)}
    nbytes = B.moe_permute_workspace_size(T, k, M)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    B.moe_permute(idx_d.data_ptr(), w_d.data_ptr(), T, k, M, out["counts"].data_ptr(), out["offsets"].data_ptr(),
                  out["slot_of"].data_ptr(), out["row_token"].data_ptr(), out["row_w"].data_ptr(), ws.data_ptr(),
                  nbytes, s)
    assert B.moe_device_status(ws.data_ptr(), s) == 0
    return out


@pytest.mark.parametrize("name,factor", [("glm_small_bf16", 1.0), ("glm_small_bf16", 0.5),
                                         ("glam_small_bf16", 0.8), ("glm_small_f32", 0.75)])
def test_capacity_drop_matches_oracle(B, name, factor):
    cfg = ms.get_config(name)
    inp = gpu_inputs(cfg)
    T, D, M, k = cfg["T"], cfg["D"], cfg["M"], cfg["k"]
    r = oracle_route(cfg, inp)
    idx, w32 = r["idx"], r["w"].astype(np.float32)
    cap = B.moe_expert_capacity(factor, T, k, M)
    ref_idx = oracle.capacity_drop(idx, M, cap)
    assert (ref_idx == M).any()                       # the case drops something
    s = torch.cuda.current_stream().cuda_stream
    idx_d = torch.as_tensor(idx, dtype=torch.int32, device="cuda")
    w_d = torch.as_tensor(w32, device="cuda")
    p = _permute(B, idx_d, w_d, T, k, M, s)
    B.moe_capacity_drop(idx_d.data_ptr(), p["slot_of"].data_ptr(), p["offsets"].data_ptr(), T, k, M, cap, s)
    torch.cuda.synchronize()
    assert np.array_equal(idx_d.cpu().numpy(), ref_idx)
    # the layer over the kept pairs
    p = _permute(B, idx_d, w_d, T, k, M, s)
    counts = p["counts"].cpu().numpy()
    assert counts.max() <= cap
    d = B.desc_from_config(cfg)
    weights = B.weights_from_tensors(inp)
    out_perm = torch.empty(T * k, D, dtype=torch.float32, device="cuda")
    wf = torch.zeros(B.moe_expert_ffn_workspace_size(d) + 256, dtype=torch.uint8, device="cuda")
    B.moe_expert_ffn(d, weights, inp["x"].data_ptr(), p["offsets"].data_ptr(), p["row_token"].data_ptr(),
                     p["row_w"].data_ptr(), out_perm.data_ptr(), wf.data_ptr(), wf.numel(), s)
    shared_out = None
    if cfg.get("I_sh"):
        shared_out = torch.empty_like(inp["x"])
        wsh = torch.zeros(B.moe_shared_expert_workspace_size(d) + 256, dtype=torch.uint8, device="cuda")
        B.moe_shared_expert(d, weights, inp["x"].data_ptr(), shared_out.data_ptr(), wsh.data_ptr(), wsh.numel(), s)
    y = torch.empty_like(inp["x"])
    B.moe_combine(d, out_perm.data_ptr(), p["slot_of"].data_ptr(),
                  None if shared_out is None else shared_out.data_ptr(), None, y.data_ptr(), s)
    torch.cuda.synchronize()
    shared = (np64(inp["sh_w1"]), np64(inp["sh_w2"])) if cfg.get("I_sh") else None
    y_ref = oracle.moe_tokens(np64(inp["x"]), ref_idx, w32.astype(np.float64), cfg["act"], HostExperts(inp),
                              shared, sentinel=M)
    check_y(dict(cfg, named=False), np64(y), y_ref)

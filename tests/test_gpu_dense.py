"""Parity of the dense FFN layer (moe_dense_ffn) and of the sparse block sum
(moe_forward_add: addend + MoE-FFN(x)) with the CPU oracle, through the C
ABI, on identical seeded inputs."""
import numpy as np
import pytest
import torch

import moe_synth as ms
import oracle
from gpu_common import check_routing, check_y, gpu_inputs, np64, oracle_route, oracle_y

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    import sparse_mixture_experts_logits_b200 as B
    return B


def dense_reference(cfg, inp, rows, with_addend):
    idx = torch.as_tensor(rows, device=inp["x"].device)
    b1, b2 = inp.get("b1"), inp.get("b2")
    return oracle.dense_layer(np64(inp["x"][idx]), cfg["act"], np64(inp["w1"]), np64(inp["w2"]),
                              None if b1 is None else np64(b1), None if b2 is None else np64(b2),
                              addend=np64(inp["addend"][idx]) if with_addend else None)


def run_dense(B, cfg, with_addend):
    inp = ms.dense_inputs(cfg, "cuda")
    layer = B.DenseLayer(cfg, inp)
    y = layer.forward(inp["x"], addend=inp["addend"] if with_addend else None)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return inp, layer, y


@pytest.mark.parametrize("with_addend", [True, False])
@pytest.mark.parametrize("name", ["glam_dense_small_bf16", "glm_dense_small_bf16", "glm_dense_small_f32",
                                  "glam_dense_small_f32"])
def test_dense_small_all_tokens(B, name, with_addend):
    cfg = ms.get_config(name)
    inp, _, y = run_dense(B, cfg, with_addend)
    rows = np.arange(cfg["T"])
    check_y(dict(cfg, named=False), np64(y), dense_reference(cfg, inp, rows, with_addend))


@pytest.mark.parametrize("over", [dict(T=1), dict(T=129), dict(T=257), dict(I=16), dict(D=16)])
def test_dense_edge_cases(B, over):
    cfg = ms.get_config("glm_dense_small_bf16", **over)
    inp, _, y = run_dense(B, cfg, True)
    check_y(dict(cfg, named=False), np64(y), dense_reference(cfg, inp, np.arange(cfg["T"]), True))


def test_dense_full_size_sampled(B):
    """The GLaM dense layer between its MoE layers (T=8192, D=2048, H=8192,
    GELU with biases) in the launch configuration the benchmark times: the
    first and last token of every 256-token tile (every tile of both GEMMs
    holds one), plus random tokens."""
    cfg = ms.get_config("glam_dense_bf16")
    inp, _, y = run_dense(B, cfg, True)
    tiles = {r for t0 in range(0, cfg["T"], 256) for r in (t0, min(t0 + 255, cfg["T"] - 1))}
    rows = np.array(sorted(tiles | set(np.random.default_rng(0).integers(0, cfg["T"], 24).tolist())))
    got = np64(y[torch.as_tensor(rows, device=y.device)])
    check_y(dict(cfg, named=False), got, dense_reference(cfg, inp, rows, True))


def test_dense_deterministic(B):
    cfg = ms.get_config("glm_dense_small_bf16")
    inp, layer, y1 = run_dense(B, cfg, True)
    y2 = layer.forward(inp["x"], addend=inp["addend"])
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("name", ["glm_small_bf16", "glam_small_bf16", "glm_small_f32"])
def test_forward_add_is_the_block_sum(B, name):
    """moe_forward_add = addend + MoE-FFN(x), the sparse block of the GLaM
    note ("Interleaving Dense and Sparse Layers"), with the same routing as
    moe_forward."""
    cfg = ms.get_config(name)
    inp = gpu_inputs(cfg)
    addend = ms.addend_tokens(cfg, "cuda")
    layer = B.MoELayer(cfg, inp)
    y = layer.forward(inp["x"], addend=addend)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    idx = layer.view("topk_idx").cpu().numpy()
    w = layer.view("topk_w").cpu().numpy()
    r = oracle_route(cfg, inp)
    w_ref, _ = check_routing(cfg, r, idx, w)
    tokens = np.arange(cfg["T"])
    y_ref = np64(addend) + oracle_y(cfg, inp, tokens, idx, w_ref)
    check_y(dict(cfg, named=False), np64(y), y_ref)
    # without the addend: the plain layer, same routing
    y0 = layer.forward(inp["x"])
    torch.cuda.synchronize()
    assert np.array_equal(layer.view("topk_idx").cpu().numpy(), idx)
    check_y(dict(cfg, named=False), np64(y0), oracle_y(cfg, inp, tokens, idx, w_ref))


def test_forward_add_requires_addend(B):
    cfg = ms.get_config("glm_small_bf16")
    inp = gpu_inputs(cfg)
    layer = B.MoELayer(cfg, inp)
    y = torch.empty_like(inp["x"])
    with pytest.raises(B.MoEError):
        B.moe_forward_add(layer.desc, layer.weights, inp["x"].data_ptr(), None, y.data_ptr(), layer.ws_ptr,
                          layer.ws_bytes, torch.cuda.current_stream().cuda_stream)

"""The expert-parallel layer (sparse_mixture_experts_logits_b200.ep) on one GPU:
world = 1, every expert local, each exchange a copy, so what runs is the
layer's compute through the C ABI in its expert-parallel order (gather into
dispatch order, a per-owner dispatch of the received rows, the experts, the
way back to arrival order, the combine).

Without a shared expert the result equals moe_forward bit for bit: the same
rows go through the same kernels in the same order.  With one, the shared
expert's output is rounded to the layer dtype before the combine, so the
layer is held to the forward's bound against the oracle.  Collected after
the forward suites (test_zzz_*)."""
import numpy as np
import pytest
import torch

import moe_synth as ms
from gpu_common import check_routing, check_y, gpu_inputs, np64, oracle_route, oracle_y

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    import sparse_mixture_experts_logits_b200 as B
    return B


def ep_layer(cfg, inp):
    from sparse_mixture_experts_logits_b200 import ep
    return ep.ExpertParallelMoE(cfg, ep.local_expert_tensors(inp, 0, 1), rank=0, world=1)


@pytest.mark.parametrize("name", ["glam_small_bf16", "glam_tiny_f32"])
def test_expert_parallel_one_rank_equals_forward(B, name):
    cfg = ms.get_config(name)
    inp = gpu_inputs(cfg)
    y_ep = ep_layer(cfg, inp).forward(inp["x"])
    y = B.MoELayer(cfg, inp).forward(inp["x"])
    torch.cuda.synchronize()
    view = torch.int16 if y.dtype == torch.bfloat16 else torch.int32
    assert torch.equal(y_ep.view(view), y.view(view))


@pytest.mark.parametrize("name", ["glm_small_bf16", "glm_grouped_bf16"])
def test_expert_parallel_one_rank_with_shared_expert(B, name):
    cfg = ms.get_config(name)
    inp = gpu_inputs(cfg)
    layer = ep_layer(cfg, inp)
    y_ep = layer.forward(inp["x"])
    ref_layer = B.MoELayer(cfg, inp)
    ref_layer.forward(inp["x"])
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    assert layer.last_plan.rows_received == cfg["T"] * cfg["k"]
    idx = ref_layer.view("topk_idx").cpu().numpy()
    w_ref, _ = check_routing(cfg, oracle_route(cfg, inp), idx, ref_layer.view("topk_w").cpu().numpy())
    tokens = np.arange(cfg["T"])
    check_y(dict(cfg, named=False), np64(y_ep), oracle_y(cfg, inp, tokens, idx, w_ref))

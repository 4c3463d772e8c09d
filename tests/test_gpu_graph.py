"""The forward pass makes no host synchronisation and no allocation, so it
can be captured once into a CUDA graph and replayed (the decode loop's way
of removing launch overhead), and it runs on any stream.  At decode sizes
the shared expert runs on the library's internal side stream: several host
threads driving layers on their own streams at once must still get the
results of one-at-a-time calls."""
import threading

import pytest
import torch

import moe_synth as ms

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    import sparse_mixture_experts_logits_b200 as B
    return B


@pytest.mark.parametrize("name", ["glm45_decode_bf16", "glam_small_bf16", "glm_grouped_bf16"])
def test_graph_replay_matches_eager(B, name):
    cfg = ms.get_config(name)
    inp = ms.layer_inputs(cfg, "cuda")
    layer = B.MoELayer(cfg, inp)
    x_static = inp["x"].clone()
    y_eager = layer.forward(x_static)          # first call also configures the kernels
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    y_static = torch.empty_like(x_static)
    with torch.cuda.graph(g, stream=side):
        layer.forward(x_static, y=y_static, stream=side)
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y_static.view(torch.int16), y_eager.view(torch.int16))
    assert layer.device_status() == 0
    # new tokens in the captured input buffer: the replay follows them
    x2 = ms.normal((cfg["T"], cfg["D"]), 1.0, ms._key(cfg, "x2"), "cuda", ms.act_dtype(cfg))
    x_static.copy_(x2)
    g.replay()
    y2_eager = layer.forward(x2)
    torch.cuda.synchronize()
    assert torch.equal(y_static.view(torch.int16), y2_eager.view(torch.int16))


def test_dense_layer_graph_replay(B):
    cfg = ms.get_config("glm_dense_small_bf16")
    inp = ms.dense_inputs(cfg, "cuda")
    layer = B.DenseLayer(cfg, inp)
    y_eager = layer.forward(inp["x"], addend=inp["addend"])
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    y_static = torch.empty_like(y_eager)
    with torch.cuda.graph(g, stream=side):
        layer.forward(inp["x"], addend=inp["addend"], y=y_static, stream=side)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y_static.view(torch.int16), y_eager.view(torch.int16))


def test_forward_on_a_side_stream(B):
    cfg = ms.get_config("glm_small_bf16")
    inp = ms.layer_inputs(cfg, "cuda")
    layer = B.MoELayer(cfg, inp)
    y0 = layer.forward(inp["x"])
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        y1 = torch.empty_like(y0)
        layer.forward(inp["x"], y=y1, stream=s)
    s.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))


def test_concurrent_decode_forwards_on_own_streams(B):
    """Two host threads, each with its own decode-size layer (shared expert,
    T * k < 4 M), workspace and stream, run forwards at the same time; the
    ctypes calls release the GIL, so the two fork to the side stream and
    join back concurrently.  Every y equals the one-at-a-time y bit for
    bit."""
    cfg = ms.get_config("glm45_decode_bf16")
    assert cfg["T"] * cfg["k"] < 4 * cfg["M"] and cfg["I_sh"] > 0
    inp = ms.layer_inputs(cfg, "cuda")
    layers = [B.MoELayer(cfg, inp), B.MoELayer(cfg, inp)]
    xs = [inp["x"], ms.normal((cfg["T"], cfg["D"]), 1.0, ms._key(cfg, "x2"), "cuda", ms.act_dtype(cfg))]
    ref = [layers[i].forward(xs[i]) for i in range(2)]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [[torch.empty_like(xs[i]) for _ in range(6)] for i in range(2)]
    for i in range(2):
        streams[i].wait_stream(torch.cuda.current_stream())
    errors = []

    def run(i):
        try:
            for y in outs[i]:
                layers[i].forward(xs[i], y=y, stream=streams[i])
        except Exception as e:  # reported below, on the main thread
            errors.append(e)

    threads = [threading.Thread(target=run, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    torch.cuda.synchronize()
    assert not errors
    for i in range(2):
        assert layers[i].device_status() == 0
        for y in outs[i]:
            assert torch.equal(y.view(torch.int16), ref[i].view(torch.int16))

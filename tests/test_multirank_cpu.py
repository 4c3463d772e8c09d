"""The N > 1 path of bench.py on CPU: two gloo ranks each take their own
slice of one global token stream (no data-path collective) and the step
time is the max over ranks."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import moe_synth as ms
    import oracle
    dist = bench.dist_init(world, rank, backend="gloo")
    cfg = ms.get_config("glm_small_bf16")
    T = 40
    r0, r1 = bench.token_rows(rank, T)
    x = ms.normal_rows(torch.arange(r0, r1), cfg["D"], 1.0, ms._key(cfg, "x"), ms.act_dtype(cfg))
    # each rank routes its own tokens with the oracle router: no exchange needed
    w_r = ms.router_weight(cfg)
    r = oracle.route(x.double().numpy(), w_r.double().numpy(), ms.router_bias(cfg).double().numpy(),
                     cfg["k"], cfg["gate"], cfg["norm_topk_prob"], cfg["alpha"], cfg["eps"])
    local_ms = 1.0 + rank * 2.5
    worst = bench.max_over_ranks(dist, local_ms, torch.device("cpu"))
    torch.save({"x": x, "idx": torch.as_tensor(r["idx"]), "worst": worst},
               os.path.join(out_dir, f"rank{rank}.pt"))
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_shard_tokens_and_take_max_time(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    sys.path.insert(0, ROOT)
    import moe_synth as ms
    import oracle
    cfg = ms.get_config("glm_small_bf16")
    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(2)]
    assert res[0]["worst"] == res[1]["worst"] == 3.5
    x_all = torch.cat([res[0]["x"], res[1]["x"]])
    # the two slices are rows 0..79 of the stream a single process would use
    full = ms.x_tokens(ms.get_config("glm_small_bf16", T=80))
    assert torch.equal(x_all.view(torch.int16), full.view(torch.int16))
    # routing of the shards equals routing of the whole batch (tokens independent)
    r = oracle.route(full.double().numpy(), ms.router_weight(cfg).double().numpy(),
                     ms.router_bias(cfg).double().numpy(), cfg["k"], cfg["gate"],
                     cfg["norm_topk_prob"], cfg["alpha"], cfg["eps"])
    assert torch.equal(torch.cat([res[0]["idx"], res[1]["idx"]]), torch.as_tensor(r["idx"]))

"""Expert parallelism's exchange on CPU gloo ranks: every rank routes its own
tokens, sends each row to the owner of its expert with the plan of
sparse_mixture_experts_logits_b200.ep, the owner computes its experts over
the rows it received, the results come back, and each rank's combine must
equal the oracle's single-process layer on that rank's tokens.

The compute steps run here in the fp64 oracle (the library's kernels need a
GPU); what is under test is the plan and the exchange: split sizes, the
arrival order and the local expert of every received row, and the way back
to each rank's dispatch order."""
import os
import socket
import sys

import numpy as np
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


def _layer_inputs(cfg):
    import moe_synth as ms
    f64 = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    return {k: f64(v) for k, v in ms.layer_inputs(cfg).items()}


def _forced_idx(T, k, M, world, rank):
    """A routing that leaves the experts of the last rank without rows and
    sends nothing from rank 0 to rank 1: every token picks k distinct experts
    among those of ranks 0 and 2.. (rank 0's tokens only among rank 0's)."""
    E = M // world
    allowed = list(range(E)) if rank == 0 else [e for e in range(M) if e // E not in (1, world - 1)]
    rng = np.random.default_rng(rank)
    return np.stack([rng.choice(allowed, size=k, replace=False) for _ in range(T)]).astype(np.int64)


def _worker(rank, world, port, name, T_total, forced, out_dir):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import moe_synth as ms
        import oracle
        from sparse_mixture_experts_logits_b200 import ep

        cfg = ms.get_config(name, T=T_total)
        inp = _layer_inputs(cfg)
        M, k, D = cfg["M"], cfg["k"], cfg["D"]
        E = ep.experts_per_rank(M, world)
        per = T_total // world
        rows = slice(rank * per, (rank + 1) * per)
        mine = dict(inp, x=inp["x"][rows])
        local_cfg = dict(cfg, T=per)
        # 1. this rank's routing and dispatch order
        if forced:
            idx = _forced_idx(per, k, M, world, rank)
            w = oracle.topk_weights(idx, mine["x"] @ inp["w_r"], oracle.sigmoid(mine["x"] @ inp["w_r"]),
                                    cfg["gate"], cfg["norm_topk_prob"], cfg["alpha"], cfg["eps"])
        else:
            r = oracle.route(mine["x"], inp["w_r"], inp.get("e_bias"), k, cfg["gate"], cfg["norm_topk_prob"],
                             cfg["alpha"], cfg["eps"])
            idx, w = r["idx"], r["w"]
        p = oracle.permute(idx, w, M)
        x_perm = torch.from_numpy(mine["x"][p["row_token"]])
        # 2. the plan and the rows out
        recv_counts = ep.exchange_counts(torch.as_tensor(p["counts"], dtype=torch.int32), world)
        plan = ep.make_plan(p["counts"], recv_counts.numpy(), world)
        assert plan.rows_sent == per * k
        x_recv = ep.send_rows(x_perm, plan)
        w_recv = ep.send_rows(torch.from_numpy(p["row_w"]), plan)
        assert x_recv.shape == (plan.rows_received, D) and w_recv.shape == (plan.rows_received,)
        # 3. this rank's experts (global ids rank*E + local) over the rows it received
        ids = ep.arrival_expert_ids(plan)
        out_arr = np.zeros((plan.rows_received, D))
        for le in np.unique(ids):
            sel = np.nonzero(ids == le)[0]
            g = rank * E + int(le)
            b1 = None if inp.get("b1") is None else inp["b1"][g]
            b2 = None if inp.get("b2") is None else inp["b2"][g]
            out = oracle.expert_ffn(x_recv.numpy()[sel], cfg["act"], inp["w1"][g], inp["w2"][g], b1, b2)
            out_arr[sel] = w_recv.numpy()[sel, None] * out
        # 4. results home, combine with the shared expert
        out_back = ep.return_rows(torch.from_numpy(out_arr), plan).numpy()
        y = np.zeros((per, D))
        for j in range(k):
            y += out_back[p["slot_of"][:, j]]
        if cfg.get("I_sh"):
            y += oracle.shared_expert(mine["x"], inp["sh_w1"], inp["sh_w2"])
        ref = oracle.moe_forward(local_cfg, mine, idx=idx)["y"]
        ok = np.allclose(y, ref, rtol=1e-12, atol=1e-12)
        total_recv = torch.tensor([plan.rows_received])
        dist.all_reduce(total_recv)
        torch.save({"ok": bool(ok), "err": float(np.abs(y - ref).max()), "recv": plan.rows_received,
                    "send": plan.send_splits, "total_recv": int(total_recv)},
                   os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("name,world,forced", [("glm_small_bf16", 2, False), ("glam_small_bf16", 4, False),
                                               ("glm_small_f32", 4, True)])
def test_expert_parallel_exchange_matches_single_process(tmp_path, name, world, forced):
    T_total = 24 * world
    mp.start_processes(_worker, args=(world, _free_port(), name, T_total, forced, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    sys.path.insert(0, ROOT)
    import moe_synth as ms
    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]
    for r, v in enumerate(res):
        assert v["ok"], (r, v["err"])
    k = ms.get_config(name)["k"]
    assert all(v["total_recv"] == T_total * k for v in res)
    if forced:
        assert res[world - 1]["recv"] == 0           # the last rank's experts got no rows
        assert res[0]["send"][1] == 0                 # rank 0 sent nothing to rank 1


def test_plan_from_a_count_matrix():
    """Rank q's plan from the counts C[s, e] that every rank s holds."""
    sys.path.insert(0, ROOT)
    from sparse_mixture_experts_logits_b200 import ep
    world, M = 3, 6
    E = M // world
    C = np.array([[1, 0, 2, 3, 0, 4], [0, 0, 5, 1, 2, 2], [7, 1, 0, 0, 0, 3]])
    for q in range(world):
        plan = ep.make_plan(C[q], C[:, q * E:(q + 1) * E], world)
        assert plan.send_splits == [int(C[q, s * E:(s + 1) * E].sum()) for s in range(world)]
        assert plan.recv_splits == [int(C[s, q * E:(q + 1) * E].sum()) for s in range(world)]
        ids = ep.arrival_expert_ids(plan)
        expect = [le for s in range(world) for le in range(E) for _ in range(C[s, q * E + le])]
        assert ids.tolist() == expect
    with pytest.raises(ValueError):
        ep.experts_per_rank(10, 4)

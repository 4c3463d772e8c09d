"""Expert parallelism on CPU gloo ranks: ExpertParallelMoE.forward (the
product's orchestration, exchange plan and collectives) with each kernel step
done by the fp64 oracle, since the library's kernels need a GPU.  Every rank
routes its own tokens, sends each row to the owner of its expert, the owner
runs its experts over the rows it received, the results come back, and each
rank's output must equal the oracle's single-process layer on its tokens.
What is under test is the plan and the exchange: split sizes, the arrival
order and the local expert of every received row, and the way back to each
rank's dispatch order."""
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


def _forced_idx(T, k, M, world, rank):
    """A routing that leaves the experts of the last rank without rows and
    sends nothing from rank 0 to rank 1: every token picks k distinct experts
    among those of ranks 0 and 2.. (rank 0's tokens only among rank 0's)."""
    E = M // world
    allowed = list(range(E)) if rank == 0 else [e for e in range(M) if e // E not in (1, world - 1)]
    rng = np.random.default_rng(rank)
    return np.stack([rng.choice(allowed, size=k, replace=False) for _ in range(T)]).astype(np.int64)


def _oracle_layer_class():
    """ExpertParallelMoE with each kernel step done by the fp64 oracle on host
    tensors; forward(), the exchange plan and the collectives are the
    product's own."""
    import oracle
    from sparse_mixture_experts_logits_b200 import ep

    class OracleEP(ep.ExpertParallelMoE):
        forced = None
        out_dtype = torch.float64

        def _route(self, x):
            c = self.cfg
            xs, w_r = x.numpy(), self.t["w_r"].numpy()
            if self.forced is not None:
                idx = self.forced
                logits = xs @ w_r
                w = oracle.topk_weights(idx, logits, oracle.sigmoid(logits), c["gate"], c["norm_topk_prob"],
                                        c["alpha"], c["eps"])
            else:
                bias = self.t.get("e_bias")
                r = oracle.route(xs, w_r, None if bias is None else bias.numpy(), c["k"], c["gate"],
                                 c["norm_topk_prob"], c["alpha"], c["eps"])
                idx, w = r["idx"], r["w"]
            return torch.as_tensor(idx, dtype=torch.int32), torch.as_tensor(w)

        def _dispatch(self, idx, tw, M):
            p = oracle.permute(idx.numpy(), tw.numpy(), M)
            return {k: torch.as_tensor(v) for k, v in p.items()}

        def _gather(self, x, p):
            return x[p["row_token"]]

        def _local_experts(self, x_recv, ids, w_recv):
            out = torch.zeros(x_recv.shape, dtype=torch.float64)
            for le in np.unique(ids):
                sel = np.nonzero(ids == le)[0]
                b1, b2 = self.t.get("b1"), self.t.get("b2")
                e = oracle.expert_ffn(x_recv.numpy()[sel], self.cfg["act"], self.t["w1"][le].numpy(),
                                      self.t["w2"][le].numpy(), None if b1 is None else b1[le].numpy(),
                                      None if b2 is None else b2[le].numpy())
                out[sel] = torch.as_tensor(w_recv.numpy()[sel, None] * e)
            return out

        def _shared(self, x):
            if not self.cfg.get("I_sh"):
                return None
            sh = oracle.shared_expert(x.numpy(), self.t["sh_w1"].numpy(), self.t["sh_w2"].numpy())
            return torch.as_tensor(sh)

        def _combine(self, out_rows, slot_of, y_sh, x):
            y = torch.zeros(x.shape, dtype=torch.float64)
            for j in range(slot_of.shape[1]):
                y += out_rows[slot_of[:, j].long()]
            return y if y_sh is None else y + y_sh

    return OracleEP


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
        full = {k: None if v is None else v.double() for k, v in ms.layer_inputs(cfg).items()}
        per = T_total // world
        x = full["x"][rank * per:(rank + 1) * per].contiguous()
        layer = _oracle_layer_class()(cfg, ep.local_expert_tensors(full, rank, world), rank, world)
        if forced:
            layer.forced = _forced_idx(per, cfg["k"], cfg["M"], world, rank)
        y = layer.forward(x).numpy()
        mine = {k: (None if v is None else v.numpy()) for k, v in full.items()}
        mine["x"] = x.numpy()
        ref = oracle.moe_forward(dict(cfg, T=per), mine, idx=layer.forced)["y"]
        plan = layer.last_plan
        total_recv = torch.tensor([plan.rows_received])
        dist.all_reduce(total_recv)
        torch.save({"ok": bool(np.allclose(y, ref, rtol=1e-12, atol=1e-12)), "err": float(np.abs(y - ref).max()),
                    "recv": plan.rows_received, "send": plan.send_splits, "total_recv": int(total_recv)},
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

"""Expert parallelism on CPU gloo ranks: ExpertParallelMoE.forward (the
product's orchestration, buffers and collectives) with each kernel step done
on the host from its definition, since the library's kernels need a GPU.
Every rank routes its own tokens, packs each expert's rows into fixed blocks
of cap rows, sends each owner its blocks with equal-split all-to-alls, the
owner runs its experts over the rows it received, the results come back, and
each rank's output must equal the oracle's single-process layer on its
tokens with the pairs past an expert's capacity dropped.  What is under test
is the fixed-split exchange: the packed layout, the arrival layout and the
way back to each token's k slots."""
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
    """ExpertParallelMoE with each kernel step done on host tensors, from the
    step's definition (the fp64 oracle for the routing, the dispatch order,
    the expert FFNs and the shared expert; the pack and the arrival layout as
    the header states them).  forward(), the buffers and the collectives are
    the product's own."""
    import oracle
    from sparse_mixture_experts_logits_b200 import ep

    class OracleEP(ep.ExpertParallelMoE):
        forced = None
        out_dtype = torch.float64
        w_dtype = torch.float64

        def _route(self, x, b):
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
            b["idx"].copy_(torch.as_tensor(idx))
            b["tw"].copy_(torch.as_tensor(w))
            self.routed = (np.asarray(idx), np.asarray(w))

        def _dispatch(self, b):
            p = oracle.permute(b["idx"].numpy(), b["tw"].numpy(), self.M)
            for name in ("counts", "offsets", "slot_of", "row_token", "row_w"):
                b[name].copy_(torch.as_tensor(p[name]).view(b[name].shape))

        def _pack(self, x, b):
            # moe_ep_pack as the header states it
            off, rt, rw = b["offsets"].numpy(), b["row_token"].numpy(), b["row_w"].numpy()
            cap = b["cap"]
            b["x_pad"].zero_()
            b["w_pad"].zero_()
            for e in range(self.M):
                n = int(off[e + 1] - off[e])
                b["kept"][e] = min(n, cap)
                for i in range(min(n, cap)):
                    b["x_pad"][e * cap + i] = x[int(rt[off[e] + i])]
                    b["w_pad"][e * cap + i] = float(rw[off[e] + i])
            so = b["slot_of"].numpy().reshape(-1)
            sp = np.full(so.shape, -1, dtype=np.int32)
            for p_, s_ in enumerate(so):
                if s_ >= 0:
                    e = int(np.searchsorted(off, s_, side="right") - 1)
                    if s_ - off[e] < cap:
                        sp[p_] = e * cap + (s_ - off[e])
            b["slot_pad"].copy_(torch.as_tensor(sp).view(b["slot_pad"].shape))

        def _local_experts(self, b):
            # arrival row (q E + e) cap + i holds local expert e's i-th row from rank q
            cap, E = b["cap"], self.E
            kept = b["recv_kept"].numpy().reshape(self.world, E)
            b["out_arr"].zero_()
            b1, b2 = self.t.get("b1"), self.t.get("b2")
            for q in range(self.world):
                for e in range(E):
                    rows = [(q * E + e) * cap + i for i in range(int(kept[q, e]))]
                    if not rows:
                        continue
                    out = oracle.expert_ffn(b["x_recv"].numpy()[rows], self.cfg["act"], self.t["w1"][e].numpy(),
                                            self.t["w2"][e].numpy(), None if b1 is None else b1[e].numpy(),
                                            None if b2 is None else b2[e].numpy())
                    b["out_arr"][rows] = torch.as_tensor(b["w_recv"].numpy()[rows, None] * out)
            self.rows_received = int(kept.sum())

        def _shared(self, x, b):
            if not self.cfg.get("I_sh"):
                return None
            return torch.as_tensor(oracle.shared_expert(x.numpy(), self.t["sh_w1"].numpy(), self.t["sh_w2"].numpy()))

        def _combine(self, b, y_sh, x):
            y = torch.zeros(x.shape, dtype=torch.float64)
            sp = b["slot_pad"]
            for j in range(sp.shape[1]):
                live = sp[:, j] >= 0
                y[live] += b["out_home"][sp[live, j].long()]
            return y if y_sh is None else y + y_sh

    return OracleEP


def _worker(rank, world, port, name, T_total, forced, factor, out_dir):
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
        layer = _oracle_layer_class()(cfg, ep.local_expert_tensors(full, rank, world), rank, world,
                                      capacity_factor=factor)
        if forced:
            layer.forced = _forced_idx(per, cfg["k"], cfg["M"], world, rank)
        y = layer.forward(x).numpy()
        mine = {k: (None if v is None else v.numpy()) for k, v in full.items()}
        mine["x"] = x.numpy()
        idx, w = layer.routed
        cap = ep.capacity(per, cfg["k"], cfg["M"], factor)
        kept_idx = oracle.capacity_drop(idx, cfg["M"], cap)
        ref = oracle.moe_forward(dict(cfg, T=per), mine, idx=kept_idx, w=w)["y"]
        n_dropped = int((kept_idx == cfg["M"]).sum())
        totals = torch.tensor([layer.rows_received, n_dropped])
        dist.all_reduce(totals)
        sent_to = layer.buffers(per, x.dtype)["kept"].view(world, -1).sum(dim=1).tolist()
        torch.save({"ok": bool(np.allclose(y, ref, rtol=1e-12, atol=1e-12)), "err": float(np.abs(y - ref).max()),
                    "recv": layer.rows_received, "send": sent_to, "total_recv": int(totals[0]),
                    "total_dropped": int(totals[1]), "cap": cap},
                   os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("name,world,forced,factor", [("glm_small_bf16", 2, False, None),
                                                      ("glam_small_bf16", 4, False, None),
                                                      ("glm_small_f32", 4, True, None),
                                                      ("glm_small_bf16", 2, False, 1.0),
                                                      ("glam_small_bf16", 4, True, 0.5)])
def test_expert_parallel_exchange_matches_single_process(tmp_path, name, world, forced, factor):
    """Each rank's y equals the oracle's single-process layer on its tokens,
    with the pairs past an expert's capacity dropped (none without a factor)."""
    T_total = 24 * world
    mp.start_processes(_worker, args=(world, _free_port(), name, T_total, forced, factor, str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    sys.path.insert(0, ROOT)
    import moe_synth as ms
    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]
    for r, v in enumerate(res):
        assert v["ok"], (r, v["err"])
    k = ms.get_config(name)["k"]
    assert all(v["total_recv"] + v["total_dropped"] == T_total * k for v in res)
    if factor is None:
        assert all(v["total_dropped"] == 0 for v in res)
    if factor is not None and factor < 1:
        assert res[0]["total_dropped"] > 0           # the capacity bites
    if forced:
        assert res[world - 1]["recv"] == 0           # the last rank's experts got no rows
        assert res[0]["send"][1] == 0                 # rank 0 sent nothing to rank 1


def test_capacity_and_split_sizes():
    """The capacity rule and the fixed split: E * cap rows per rank pair,
    whatever the routing."""
    sys.path.insert(0, ROOT)
    from sparse_mixture_experts_logits_b200 import ep
    assert ep.capacity(24, 2, 8, None) == 24
    assert ep.capacity(24, 2, 8, 1.0) == 6                 # ceil(24 * 2 / 8)
    assert ep.capacity(24, 2, 8, 1.1) == 7
    assert ep.capacity(24, 2, 8, 100.0) == 24              # never above T
    assert ep.capacity(0, 2, 8, 1.0) == 0
    with pytest.raises(ValueError):
        ep.capacity(24, 2, 8, -1.0)
    with pytest.raises(ValueError):
        ep.experts_per_rank(10, 4)

"""Expert parallelism: the routed experts of one layer split over the ranks
of a process group, the tokens of each rank sent to the experts' owners and
their outputs sent back.

The pages name the cost this layout pays: experts spread over machines make
every routing decision a transfer of token rows and results (the GLaM
industry article, the first route: cross-node communication between expert
"buildings"; the second route: fine-grained expert parallelism).  The layer
itself is unchanged: rank q owns experts [q E, (q + 1) E), E = M / world;
every rank keeps the router and the shared expert.

One forward on each rank, in the order the ranks run it:
  1. route and dispatch its own tokens (moe_route_topk, moe_permute), and
     copy its rows into dispatch order (moe_gather_rows); the dispatch order
     is expert-major, so the rows for each owner are one contiguous piece;
  2. exchange the per-expert row counts (all-to-all of M int32), then the
     rows and their gate weights (all-to-all with those split sizes);
  3. run its E experts over the rows it received (moe_permute by local
     expert, moe_expert_ffn: out = w * E_e(x), fp32), and put the results
     back in arrival order (moe_combine with k = 1, fp32);
  4. send the results back (all-to-all, the splits reversed), which leaves
     each rank its own rows in its own dispatch order, and combine them with
     its shared expert (moe_shared_expert, moe_combine).

The exchange plan (step 2) is plain host logic on the counts and is what the
CPU tests check with gloo ranks; the compute steps are the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import abi
from .layer import _ptr, _stream_handle, desc_from_config


def experts_per_rank(M: int, world: int) -> int:
    if world < 1 or M % world != 0:
        raise ValueError(f"{M} experts do not split evenly over {world} ranks")
    return M // world


@dataclass
class ExchangePlan:
    """Row counts of one exchange.  send_splits[q]: rows this rank sends to
    rank q (its experts' rows, contiguous in dispatch order); recv_counts[s, e]:
    rows rank s sends for this rank's local expert e; recv_splits[s]: their sum."""
    send_splits: list
    recv_splits: list
    recv_counts: np.ndarray

    @property
    def rows_received(self) -> int:
        return int(sum(self.recv_splits))

    @property
    def rows_sent(self) -> int:
        return int(sum(self.send_splits))


def exchange_counts(counts: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """All-to-all of the per-expert counts [M] (int32): rank q receives, from
    every rank s, the counts of q's own experts, as [world, E]."""
    import torch.distributed as dist

    E = experts_per_rank(counts.numel(), world)
    recv = torch.empty_like(counts)
    if world == 1:
        recv.copy_(counts)
    else:
        dist.all_to_all_single(recv, counts.contiguous(), group=group)
    return recv.view(world, E)


def make_plan(counts_host, recv_counts_host, world: int) -> ExchangePlan:
    counts_host = np.asarray(counts_host, dtype=np.int64)
    E = experts_per_rank(counts_host.size, world)
    recv = np.asarray(recv_counts_host, dtype=np.int64).reshape(world, E)
    send = counts_host.reshape(world, E).sum(axis=1)
    return ExchangePlan([int(v) for v in send], [int(v) for v in recv.sum(axis=1)], recv)


def arrival_expert_ids(plan: ExchangePlan) -> np.ndarray:
    """Local expert of every received row, in arrival order: from each
    source rank in turn, its rows for local experts 0..E-1 in that order."""
    world, E = plan.recv_counts.shape
    ids = np.tile(np.arange(E, dtype=np.int32), world)
    return np.repeat(ids, plan.recv_counts.reshape(-1))


def send_rows(rows: torch.Tensor, plan: ExchangePlan, group=None) -> torch.Tensor:
    """Rows in dispatch order out to their experts' owners; returns the rows
    received, in arrival order."""
    import torch.distributed as dist

    out = torch.empty((plan.rows_received,) + tuple(rows.shape[1:]), dtype=rows.dtype, device=rows.device)
    if len(plan.send_splits) == 1:
        out.copy_(rows[:plan.rows_sent])
    else:
        dist.all_to_all_single(out, rows[:plan.rows_sent].contiguous(), output_split_sizes=plan.recv_splits,
                               input_split_sizes=plan.send_splits, group=group)
    return out


def return_rows(rows: torch.Tensor, plan: ExchangePlan, group=None) -> torch.Tensor:
    """Results in arrival order back to the ranks that sent the rows; returns
    this rank's rows in its own dispatch order."""
    import torch.distributed as dist

    out = torch.empty((plan.rows_sent,) + tuple(rows.shape[1:]), dtype=rows.dtype, device=rows.device)
    if len(plan.send_splits) == 1:
        out.copy_(rows)
    else:
        dist.all_to_all_single(out, rows.contiguous(), output_split_sizes=plan.send_splits,
                               input_split_sizes=plan.recv_splits, group=group)
    return out


def local_expert_tensors(tensors: dict, rank: int, world: int) -> dict:
    """This rank's slice of the routed experts' weights; router and shared
    expert whole."""
    M = tensors["w1"].shape[0]
    E = experts_per_rank(M, world)
    out = dict(tensors)
    for k in ("w1", "w2", "b1", "b2"):
        if tensors.get(k) is not None:
            out[k] = tensors[k][rank * E:(rank + 1) * E].contiguous()
    return out


class ExpertParallelMoE:
    """One MoE layer with its routed experts split over ``world`` ranks.

    ``tensors`` holds the router (w_r, e_bias), THIS rank's experts
    (w1/w2/b1/b2 with E = M / world rows each, see local_expert_tensors) and
    the shared expert, all on this rank's device."""

    def __init__(self, cfg: dict, tensors: dict, rank: int, world: int, group=None):
        self.cfg = cfg
        self.rank, self.world, self.group = rank, world, group
        self.M = cfg["M"]
        self.E = experts_per_rank(self.M, world)
        if tensors["w1"].shape[0] != self.E:
            raise ValueError("tensors must hold this rank's experts only")
        self.t = tensors
        self.device = tensors["w_r"].device
        self.w_local = abi.Weights()
        for name in ("w1", "b1", "w2", "b2"):
            setattr(self.w_local, name, _ptr(tensors.get(name)))
        self.w_shared = abi.Weights()
        self.w_shared.sh_w1, self.w_shared.sh_w2 = _ptr(tensors.get("sh_w1")), _ptr(tensors.get("sh_w2"))

    def launch_count(self, T: int, rows_received: int) -> int:
        """Kernels of the library one forward on this rank launches (the
        collectives' own kernels not counted)."""
        bf16 = self.cfg["dtype"] == "bf16"
        k = self.cfg["k"]
        n = 3 if bf16 else 2                                  # router logits + top-k
        n += 1 if T * k <= 2048 else 3                        # dispatch order
        n += 1                                                # rows into dispatch order
        if rows_received > 0:
            n += 1 if rows_received <= 2048 else 3            # received rows by local expert
            n += 3 if bf16 else 2                             # [gather,] the expert GEMMs
            n += 1                                            # back to arrival order
        n += 2 if self.cfg.get("I_sh") else 0                 # shared expert
        return n + 1                                          # combine

    def _desc(self, T, M=None, k=None, dtype=None):
        d = desc_from_config(self.cfg, T)
        if M is not None:
            d.M, d.n_group, d.topk_group = M, 1, 1
        if k is not None:
            d.k = k
        if dtype is not None:
            d.dtype = dtype
        return d

    @staticmethod
    def _ws(nbytes, device):
        buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        return buf, buf.data_ptr() + (-buf.data_ptr()) % 256

    def forward(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        cfg, dev = self.cfg, self.device
        T, D = x.shape
        M, k = self.M, cfg["k"]
        s = _stream_handle(stream)
        d = self._desc(T)
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        status = torch.zeros(1, **i32)
        # 1. route and dispatch this rank's tokens
        idx = torch.empty((T, k), **i32)
        tw = torch.empty((T, k), **f32)
        rbuf, rws = self._ws(abi.moe_route_workspace_size(T, D, M, d.dtype), dev)
        abi.moe_route_topk(x.data_ptr(), _ptr(self.t["w_r"]), _ptr(self.t.get("e_bias")), T, D, M, k, d.dtype,
                           d.gate, d.norm_topk_prob, d.routed_scaling_factor, d.eps, d.n_group, d.topk_group,
                           idx.data_ptr(), tw.data_ptr(), rws, rbuf.numel() - 256, s)
        counts = torch.empty(M, **i32)
        offsets = torch.empty(M + 1, **i32)
        slot_of = torch.empty((T, k), **i32)
        row_token = torch.empty(T * k, **i32)
        row_w = torch.empty(T * k, **f32)
        pbuf, pws = self._ws(abi.moe_permute_workspace_size(T, k, M), dev)
        abi.moe_permute(idx.data_ptr(), tw.data_ptr(), T, k, M, counts.data_ptr(), offsets.data_ptr(),
                        slot_of.data_ptr(), row_token.data_ptr(), row_w.data_ptr(), pws, pbuf.numel() - 256, s)
        x_perm = torch.empty((T * k, D), dtype=x.dtype, device=dev)
        abi.moe_gather_rows(x.data_ptr(), row_token.data_ptr(), offsets[M:].data_ptr(), x_perm.data_ptr(), T * k,
                            T, D, d.dtype, status.data_ptr(), s)
        # 2. the exchange plan and the rows out
        recv_counts = exchange_counts(counts, self.world, self.group)
        plan = make_plan(counts.cpu().numpy(), recv_counts.cpu().numpy(), self.world)
        x_recv = send_rows(x_perm, plan, self.group)
        w_recv = send_rows(row_w, plan, self.group)
        # 3. this rank's experts over the rows it received
        R = plan.rows_received
        out_arr = torch.empty((R, D), **f32)
        if R > 0:
            ids = torch.as_tensor(arrival_expert_ids(plan), device=dev).view(R, 1)
            l_counts = torch.empty(self.E, **i32)
            l_offsets = torch.empty(self.E + 1, **i32)
            l_slot = torch.empty((R, 1), **i32)
            l_token = torch.empty(R, **i32)
            l_w = torch.empty(R, **f32)
            lbuf, lws = self._ws(abi.moe_permute_workspace_size(R, 1, self.E), dev)
            abi.moe_permute(ids.data_ptr(), w_recv.data_ptr(), R, 1, self.E, l_counts.data_ptr(),
                            l_offsets.data_ptr(), l_slot.data_ptr(), l_token.data_ptr(), l_w.data_ptr(), lws,
                            lbuf.numel() - 256, s)
            d_loc = self._desc(R, M=self.E, k=1)
            out_perm = torch.empty((R, D), **f32)
            fbuf, fws = self._ws(abi.moe_expert_ffn_workspace_size(d_loc), dev)
            abi.moe_expert_ffn(d_loc, self.w_local, x_recv.data_ptr(), l_offsets.data_ptr(), l_token.data_ptr(),
                               l_w.data_ptr(), out_perm.data_ptr(), fws, fbuf.numel() - 256, s)
            # back to arrival order: row r is the (only) slot of "token" r
            abi.moe_combine(self._desc(R, M=self.E, k=1, dtype=abi.DTYPE_F32), out_perm.data_ptr(),
                            l_slot.data_ptr(), None, None, out_arr.data_ptr(), s)
        # 4. results home, then this rank's combine with its shared expert
        out_back = return_rows(out_arr, plan, self.group)
        y_sh = None
        if cfg.get("I_sh"):
            y_sh = torch.empty_like(x)
            sbuf, sws = self._ws(abi.moe_shared_expert_workspace_size(d), dev)
            abi.moe_shared_expert(d, self.w_shared, x.data_ptr(), y_sh.data_ptr(), sws, sbuf.numel() - 256, s)
        # the router never picks the sentinel, so every one of the T k pairs went out and came back
        assert plan.rows_sent == T * k
        y = torch.empty_like(x)
        abi.moe_combine(d, out_back.data_ptr(), slot_of.data_ptr(), _ptr(y_sh), None, y.data_ptr(), s)
        self.last_plan = plan
        self.status = status
        return y

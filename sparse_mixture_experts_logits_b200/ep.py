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

    out_dtype = torch.float32  # the experts' outputs as they travel back (moe_expert_ffn's fp32 rows)

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

    # ---- the library's kernels, one method per step (tensors in, tensors out) ----

    def _route(self, x):
        """topk_idx [T, k] int32 and topk_w [T, k] fp32 (moe_route_topk)."""
        T, D = x.shape
        M, k = self.M, self.cfg["k"]
        d = self._desc(T)
        idx = torch.empty((T, k), dtype=torch.int32, device=self.device)
        tw = torch.empty((T, k), dtype=torch.float32, device=self.device)
        buf, ws = self._ws(abi.moe_route_workspace_size(T, D, M, d.dtype), self.device)
        abi.moe_route_topk(x.data_ptr(), _ptr(self.t["w_r"]), _ptr(self.t.get("e_bias")), T, D, M, k, d.dtype,
                           d.gate, d.norm_topk_prob, d.routed_scaling_factor, d.eps, d.n_group, d.topk_group,
                           idx.data_ptr(), tw.data_ptr(), ws, buf.numel() - 256, self._s)
        return idx, tw

    def _dispatch(self, idx, tw, M):
        """The dispatch order of (idx, tw) over M experts (moe_permute)."""
        T, k = idx.shape
        i32 = dict(dtype=torch.int32, device=self.device)
        p = {"counts": torch.empty(M, **i32), "offsets": torch.empty(M + 1, **i32),
             "slot_of": torch.empty((T, k), **i32), "row_token": torch.empty(T * k, **i32),
             "row_w": torch.empty(T * k, dtype=torch.float32, device=self.device)}
        buf, ws = self._ws(abi.moe_permute_workspace_size(T, k, M), self.device)
        abi.moe_permute(idx.data_ptr(), tw.data_ptr(), T, k, M, p["counts"].data_ptr(), p["offsets"].data_ptr(),
                        p["slot_of"].data_ptr(), p["row_token"].data_ptr(), p["row_w"].data_ptr(), ws,
                        buf.numel() - 256, self._s)
        return p

    def _gather(self, x, p):
        """x's rows in dispatch order (moe_gather_rows)."""
        T, D = x.shape
        rows = p["row_token"].numel()
        out = torch.empty((rows, D), dtype=x.dtype, device=self.device)
        abi.moe_gather_rows(x.data_ptr(), p["row_token"].data_ptr(), p["offsets"][self.M:].data_ptr(),
                            out.data_ptr(), rows, T, D, self._desc(T).dtype, self.status.data_ptr(), self._s)
        return out

    def _local_experts(self, x_recv, ids, w_recv):
        """w * E_e(x) (fp32) of every received row, in arrival order: the rows
        ordered by local expert (moe_permute, k = 1), the experts
        (moe_expert_ffn), and back to arrival order (moe_combine, k = 1, fp32)."""
        R, D = x_recv.shape
        out_arr = torch.empty((R, D), dtype=torch.float32, device=self.device)
        ids_d = torch.as_tensor(ids, device=self.device).view(R, 1)
        p = self._dispatch(ids_d, w_recv.view(R, 1), self.E)
        d_loc = self._desc(R, M=self.E, k=1)
        out_perm = torch.empty((R, D), dtype=torch.float32, device=self.device)
        buf, ws = self._ws(abi.moe_expert_ffn_workspace_size(d_loc), self.device)
        abi.moe_expert_ffn(d_loc, self.w_local, x_recv.data_ptr(), p["offsets"].data_ptr(),
                           p["row_token"].data_ptr(), p["row_w"].data_ptr(), out_perm.data_ptr(), ws,
                           buf.numel() - 256, self._s)
        # row r is the only slot of "token" r
        abi.moe_combine(self._desc(R, M=self.E, k=1, dtype=abi.DTYPE_F32), out_perm.data_ptr(),
                        p["slot_of"].data_ptr(), None, None, out_arr.data_ptr(), self._s)
        return out_arr

    def _shared(self, x):
        """The shared expert's output in the layer dtype, or None."""
        if not self.cfg.get("I_sh"):
            return None
        d = self._desc(x.shape[0])
        y_sh = torch.empty_like(x)
        buf, ws = self._ws(abi.moe_shared_expert_workspace_size(d), self.device)
        abi.moe_shared_expert(d, self.w_shared, x.data_ptr(), y_sh.data_ptr(), ws, buf.numel() - 256, self._s)
        return y_sh

    def _combine(self, out_rows, slot_of, y_sh, x):
        """y[t] = sum_j out_rows[slot_of[t, j]] (+ y_sh[t]) (moe_combine)."""
        y = torch.empty_like(x)
        abi.moe_combine(self._desc(x.shape[0]), out_rows.data_ptr(), slot_of.data_ptr(), _ptr(y_sh), None,
                        y.data_ptr(), self._s)
        return y

    # ---- one forward ----

    def forward(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        T = x.shape[0]
        k = self.cfg["k"]
        self._s = _stream_handle(stream) if x.is_cuda else None
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        # 1. route and dispatch this rank's tokens; its rows in dispatch order
        idx, tw = self._route(x)
        p = self._dispatch(idx, tw, self.M)
        x_perm = self._gather(x, p)
        # 2. the exchange plan and the rows out
        recv_counts = exchange_counts(p["counts"], self.world, self.group)
        plan = make_plan(p["counts"].cpu().numpy(), recv_counts.cpu().numpy(), self.world)
        # the router never picks the sentinel, so all T k pairs go out and come back
        assert plan.rows_sent == T * k
        x_recv = send_rows(x_perm, plan, self.group)
        w_recv = send_rows(p["row_w"], plan, self.group)
        # 3. this rank's experts over the rows it received
        if plan.rows_received > 0:
            out_arr = self._local_experts(x_recv, arrival_expert_ids(plan), w_recv)
        else:
            out_arr = torch.empty((0, x.shape[1]), dtype=self.out_dtype, device=self.device)
        # 4. results home, then this rank's combine with its shared expert
        out_back = return_rows(out_arr, plan, self.group)
        y = self._combine(out_back, p["slot_of"], self._shared(x), x)
        self.last_plan = plan
        return y

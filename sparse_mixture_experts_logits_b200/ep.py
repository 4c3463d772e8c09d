"""Expert parallelism: the routed experts of one layer split over the ranks
of a process group, the tokens of each rank sent to the experts' owners and
their outputs sent back.

The pages name the cost this layout pays: experts spread over machines make
every routing decision a transfer of token rows and results (the GLaM
industry article, the first route: cross-node communication between expert
"buildings"; the second route: fine-grained expert parallelism).  The layer
itself is unchanged: rank q owns experts [q E, (q + 1) E), E = M / world;
every rank keeps the router and the shared expert.

The exchange has fixed split sizes.  Each expert takes at most ``cap`` rows
from each rank (moe_expert_capacity; with no capacity factor, cap = T and
nothing is ever dropped), and every rank sends every other rank exactly
E * cap rows, padding included.  So no row count has to reach the host: a
step issues its kernels and collectives back to back with no
device-to-host read.  All buffers are allocated once per token count.

One forward on each rank, in the order the ranks run it:
  1. route and dispatch its own tokens (moe_route_topk, moe_permute) and
     pack its rows into M blocks of cap rows (moe_ep_pack): owner q's
     blocks are one contiguous piece, padding rows zero with weight 0;
  2. exchange the blocks' kept-row counts, the rows and their gate weights
     (three all-to-alls of equal splits);
  3. turn the [world][E][cap] arrival blocks into an expert-major dispatch
     (moe_ep_unpack), run its E experts (moe_expert_ffn: w * E_e(x), fp32)
     and put the results back into arrival order (moe_combine, k = 1, fp32;
     padding rows come out zero);
  4. send the results back (an all-to-all of equal splits), which leaves
     each rank its own rows in its own packed layout, and combine them with
     its shared expert (moe_shared_expert, moe_combine over the packed slots;
     a pair dropped by the capacity adds nothing).

The compute steps are the library's kernels.  The orchestration and the
collectives are what the CPU tests run on gloo ranks, with each kernel step
replaced by the fp64 oracle.
"""
from __future__ import annotations

import torch

from . import abi
from .layer import _ptr, _stream_handle, desc_from_config


def experts_per_rank(M: int, world: int) -> int:
    if world < 1 or M % world != 0:
        raise ValueError(f"{M} experts do not split evenly over {world} ranks")
    return M // world


def capacity(T: int, k: int, M: int, factor: float | None) -> int:
    """Rows an expert takes from one rank: moe_expert_capacity's
    ceil(factor * T * k / M), capped at T (a token picks an expert at most
    once), or T without a factor: every pair kept."""
    if factor is None:
        return T
    c = abi.moe_expert_capacity(factor, T, k, M)
    if c < 0:
        raise ValueError(f"bad capacity factor {factor}")
    return min(T, c)


def all_to_all_equal(out: torch.Tensor, inp: torch.Tensor, world: int, group=None) -> None:
    """out[q-th piece] on every rank = piece q of rank s's inp, pieces of equal
    size along dim 0 (no split sizes: nothing about the routing is needed)."""
    if world == 1:
        out.copy_(inp)
        return
    import torch.distributed as dist
    dist.all_to_all_single(out, inp, group=group)


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
    the shared expert, all on this rank's device.  ``capacity_factor``: each
    expert takes at most ceil(factor * T * k / M) rows from each rank (the
    first ones in dispatch order, as moe_capacity_drop); None keeps every
    pair, at the cost of M * T rows of send buffer."""

    out_dtype = torch.float32  # the experts' outputs as they travel back (moe_expert_ffn's fp32 rows)
    w_dtype = torch.float32    # gate weights (the ABI's fp32)

    def __init__(self, cfg: dict, tensors: dict, rank: int, world: int, group=None,
                 capacity_factor: float | None = None):
        self.cfg = cfg
        self.rank, self.world, self.group = rank, world, group
        self.M = cfg["M"]
        self.k = cfg["k"]
        self.E = experts_per_rank(self.M, world)
        if tensors["w1"].shape[0] != self.E:
            raise ValueError("tensors must hold this rank's experts only")
        self.t = tensors
        self.device = tensors["w_r"].device
        self.capacity_factor = capacity_factor
        self.w_local = abi.Weights()
        for name in ("w1", "b1", "w2", "b2"):
            setattr(self.w_local, name, _ptr(tensors.get(name)))
        self.w_shared = abi.Weights()
        self.w_shared.sh_w1, self.w_shared.sh_w2 = _ptr(tensors.get("sh_w1")), _ptr(tensors.get("sh_w2"))
        self._bufs = {}
        # device error words (MOE_DEVERR_*): [0] the pack, [1] the unpack
        self.status = torch.zeros(2, dtype=torch.int32, device=self.device)

    def launch_count(self, T: int) -> int:
        """Kernels of the library one forward on this rank launches (the
        collectives' own kernels not counted)."""
        bf16 = self.cfg["dtype"] == "bf16"
        n = 3 if bf16 else 2                                  # router logits + top-k
        n += 1 if T * self.k <= 2048 else 3                   # dispatch order
        n += 2                                                # pack rows, packed slots
        n += 1                                                # arrival blocks -> dispatch order
        n += 3 if bf16 else 2                                 # [gather,] the expert GEMMs
        n += 1                                                # back to arrival order
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

    def buffers(self, T: int, x_dtype: torch.dtype) -> dict:
        """Every tensor and workspace one forward over T tokens uses, made on
        the first call with that T and reused after."""
        key = (T, x_dtype)
        if key in self._bufs:
            return self._bufs[key]
        M, k, E, world, D = self.M, self.k, self.E, self.world, self.cfg["D"]
        cap = capacity(T, k, M, self.capacity_factor)
        R = world * E * cap                                   # rows sent = rows received
        dev = self.device
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=self.w_dtype, device=dev)
        b = {"cap": cap, "R": R,
             "idx": torch.empty((T, k), **i32), "tw": torch.empty((T, k), **f32),
             "counts": torch.empty(M, **i32), "offsets": torch.empty(M + 1, **i32),
             "slot_of": torch.empty((T, k), **i32), "row_token": torch.empty(T * k, **i32),
             "row_w": torch.empty(T * k, **f32),
             "x_pad": torch.empty((R, D), dtype=x_dtype, device=dev), "w_pad": torch.empty(R, **f32),
             "slot_pad": torch.empty((T, k), **i32), "kept": torch.empty(M, **i32),
             "x_recv": torch.empty((R, D), dtype=x_dtype, device=dev), "w_recv": torch.empty(R, **f32),
             "recv_kept": torch.empty(M, **i32),
             "loc_offsets": torch.empty(E + 1, **i32), "loc_row_token": torch.empty(max(R, 1), **i32),
             "loc_row_w": torch.empty(max(R, 1), **f32), "loc_slot": torch.empty(max(R, 1), **i32),
             "out_perm": torch.empty((R, D), dtype=self.out_dtype, device=dev),
             "out_arr": torch.empty((R, D), dtype=self.out_dtype, device=dev),
             "out_home": torch.empty((R, D), dtype=self.out_dtype, device=dev),
             "y_sh": torch.empty((T, D), dtype=x_dtype, device=dev) if self.cfg.get("I_sh") else None,
             "y": torch.empty((T, D), dtype=x_dtype, device=dev)}
        if dev.type == "cuda":
            dt = self._desc(T).dtype
            b["ws_route"] = self._ws(abi.moe_route_workspace_size(T, D, M, dt), dev)
            b["ws_perm"] = self._ws(abi.moe_permute_workspace_size(T, k, M), dev)
            b["ws_ffn"] = self._ws(abi.moe_expert_ffn_workspace_size(self._desc(R, M=E, k=1)), dev)
            if self.cfg.get("I_sh"):
                b["ws_sh"] = self._ws(abi.moe_shared_expert_workspace_size(self._desc(T)), dev)
        self._bufs[key] = b
        return b

    # ---- the library's kernels, one method per step ----

    def _route(self, x, b):
        """topk_idx [T, k] int32 and topk_w [T, k] fp32 (moe_route_topk)."""
        T, D = x.shape
        d = self._desc(T)
        buf, ws = b["ws_route"]
        abi.moe_route_topk(x.data_ptr(), _ptr(self.t["w_r"]), _ptr(self.t.get("e_bias")), T, D, self.M, self.k,
                           d.dtype, d.gate, d.norm_topk_prob, d.routed_scaling_factor, d.eps, d.n_group,
                           d.topk_group, b["idx"].data_ptr(), b["tw"].data_ptr(), ws, buf.numel() - 256, self._s)

    def _dispatch(self, b):
        """The dispatch order of (idx, tw) over the M experts (moe_permute)."""
        T, k = b["idx"].shape
        buf, ws = b["ws_perm"]
        abi.moe_permute(b["idx"].data_ptr(), b["tw"].data_ptr(), T, k, self.M, b["counts"].data_ptr(),
                        b["offsets"].data_ptr(), b["slot_of"].data_ptr(), b["row_token"].data_ptr(),
                        b["row_w"].data_ptr(), ws, buf.numel() - 256, self._s)

    def _pack(self, x, b):
        """x_pad, w_pad, slot_pad and kept from the dispatch order (moe_ep_pack)."""
        T, D = x.shape
        abi.moe_ep_pack(x.data_ptr(), b["offsets"].data_ptr(), b["row_token"].data_ptr(), b["row_w"].data_ptr(),
                        b["slot_of"].data_ptr(), T, self.k, self.M, D, self._desc(T).dtype, b["cap"],
                        b["x_pad"].data_ptr(), b["w_pad"].data_ptr(), b["slot_pad"].data_ptr(),
                        b["kept"].data_ptr(), self.status[0:1].data_ptr(), self._s)

    def _local_experts(self, b):
        """out_arr: w * E_e(x) (fp32) of every arrival row, zero on padding:
        the arrival blocks in expert-major order (moe_ep_unpack), the experts
        (moe_expert_ffn), and back to arrival order (moe_combine, k = 1)."""
        R, E = b["R"], self.E
        if R == 0:
            return
        abi.moe_ep_unpack(b["recv_kept"].data_ptr(), b["w_recv"].data_ptr(), self.world, E, b["cap"],
                          b["loc_offsets"].data_ptr(), b["loc_row_token"].data_ptr(), b["loc_row_w"].data_ptr(),
                          b["loc_slot"].data_ptr(), self.status[1:2].data_ptr(), self._s)
        d_loc = self._desc(R, M=E, k=1)
        buf, ws = b["ws_ffn"]
        abi.moe_expert_ffn(d_loc, self.w_local, b["x_recv"].data_ptr(), b["loc_offsets"].data_ptr(),
                           b["loc_row_token"].data_ptr(), b["loc_row_w"].data_ptr(), b["out_perm"].data_ptr(), ws,
                           buf.numel() - 256, self._s)
        abi.moe_combine(self._desc(R, M=E, k=1, dtype=abi.DTYPE_F32), b["out_perm"].data_ptr(),
                        b["loc_slot"].data_ptr(), None, None, b["out_arr"].data_ptr(), self._s)

    def _shared(self, x, b):
        """The shared expert's output in the layer dtype, or None."""
        if not self.cfg.get("I_sh"):
            return None
        buf, ws = b["ws_sh"]
        abi.moe_shared_expert(self._desc(x.shape[0]), self.w_shared, x.data_ptr(), b["y_sh"].data_ptr(), ws,
                              buf.numel() - 256, self._s)
        return b["y_sh"]

    def _combine(self, b, y_sh, x):
        """y[t] = sum_j out_home[slot_pad[t, j]] (+ y_sh[t]) (moe_combine)."""
        abi.moe_combine(self._desc(x.shape[0]), b["out_home"].data_ptr(), b["slot_pad"].data_ptr(), _ptr(y_sh),
                        None, b["y"].data_ptr(), self._s)
        return b["y"]

    # ---- one forward ----

    def forward(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        """y for this rank's tokens.  The returned tensor is a buffer reused by
        the next forward with the same token count."""
        T = x.shape[0]
        self._s = _stream_handle(stream) if x.is_cuda else None
        b = self.buffers(T, x.dtype)
        # 1. route, dispatch and pack this rank's tokens
        self._route(x, b)
        self._dispatch(b)
        self._pack(x, b)
        # 2. kept counts, rows and gate weights out: every split is E * cap rows
        all_to_all_equal(b["recv_kept"], b["kept"], self.world, self.group)
        all_to_all_equal(b["x_recv"], b["x_pad"], self.world, self.group)
        all_to_all_equal(b["w_recv"], b["w_pad"], self.world, self.group)
        # 3. this rank's experts over the rows it received
        self._local_experts(b)
        # 4. results home, then this rank's combine with its shared expert
        all_to_all_equal(b["out_home"], b["out_arr"], self.world, self.group)
        return self._combine(b, self._shared(x, b), x)

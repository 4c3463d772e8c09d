"""Torch-side convenience around the C ABI: descriptor and weight structs
from tensors, a workspace buffer, and views of the intermediates that
moe_forward leaves in it.  No computation happens here."""
from __future__ import annotations

import torch

from . import abi

_GATES = {"softmax": abi.GATE_SOFTMAX, "sigmoid_bias": abi.GATE_SIGMOID_BIAS}
_ACTS = {"gelu_tanh": abi.ACT_GELU_TANH, "swiglu": abi.ACT_SWIGLU}
_DTYPES = {"f32": abi.DTYPE_F32, "bf16": abi.DTYPE_BF16}


def desc_from_config(cfg: dict, T: int | None = None) -> abi.LayerDesc:
    d = abi.LayerDesc()
    d.dtype = _DTYPES[cfg["dtype"]]
    d.T = cfg["T"] if T is None else T
    d.D, d.M, d.k, d.I = cfg["D"], cfg["M"], cfg["k"], cfg["I"]
    d.gate = _GATES[cfg["gate"]]
    d.act = _ACTS[cfg["act"]]
    d.has_bias = int(bool(cfg.get("has_bias", 0)))
    d.norm_topk_prob = int(bool(cfg.get("norm_topk_prob", 1)))
    d.routed_scaling_factor = float(cfg.get("alpha", 1.0))
    d.eps = float(cfg.get("eps", 1e-20))
    d.I_sh = int(cfg.get("I_sh", 0) or 0)
    d.n_group = int(cfg.get("n_group", 1) or 1)
    d.topk_group = int(cfg.get("topk_group", 1) or 1)
    return d


def dense_desc_from_config(cfg: dict, T: int | None = None) -> abi.DenseDesc:
    d = abi.DenseDesc()
    d.dtype = _DTYPES[cfg["dtype"]]
    d.T = cfg["T"] if T is None else T
    d.D, d.I = cfg["D"], cfg["I"]
    d.act = _ACTS[cfg["act"]]
    d.has_bias = int(bool(cfg.get("has_bias", 0)))
    return d


def _ptr(t):
    return None if t is None else t.data_ptr()


def weights_from_tensors(t: dict) -> abi.Weights:
    w = abi.Weights()
    for name in ("w_r", "e_bias", "w1", "b1", "w2", "b2", "sh_w1", "sh_w2"):
        v = t.get(name)
        if v is not None and not v.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        setattr(w, name, _ptr(v))
    return w


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


class MoELayer:
    """One MoE layer bound to device weight tensors (kept alive here)."""

    def __init__(self, cfg: dict, tensors: dict, T: int | None = None):
        self.cfg = cfg
        self.tensors = tensors
        self.desc = desc_from_config(cfg, T)
        self.weights = weights_from_tensors(tensors)
        self.device = tensors["w_r"].device
        self.ws_bytes = abi.moe_workspace_size(self.desc)
        if self.ws_bytes == 0:
            raise abi.MoEError("moe_workspace_size", abi.MOE_ERR_INVALID_ARG)
        self.ws = torch.zeros(self.ws_bytes + 256, dtype=torch.uint8, device=self.device)
        base = self.ws.data_ptr()
        self._ws_off = (-base) % 256
        self.layout = abi.moe_workspace_layout(self.desc)
        self._bws = None

    @property
    def ws_ptr(self) -> int:
        return self.ws.data_ptr() + self._ws_off

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, stream=None,
                addend: torch.Tensor | None = None) -> torch.Tensor:
        """y = MoE-FFN(x), or addend + MoE-FFN(x) when ``addend`` is given."""
        if y is None:
            y = torch.empty_like(x)
        if addend is None:
            abi.moe_forward(self.desc, self.weights, x.data_ptr(), y.data_ptr(), self.ws_ptr, self.ws_bytes,
                            _stream_handle(stream))
        else:
            abi.moe_forward_add(self.desc, self.weights, x.data_ptr(), addend.data_ptr(), y.data_ptr(),
                                self.ws_ptr, self.ws_bytes, _stream_handle(stream))
        return y

    def device_status(self, stream=None) -> int:
        return abi.moe_device_status(self.ws_ptr, _stream_handle(stream))

    def grad_shapes(self) -> dict:
        """Shapes of the gradients moe_backward writes (None: not written)."""
        d = self.desc
        swiglu = d.act == abi.ACT_SWIGLU
        n1 = 2 * d.I if swiglu else d.I
        biases = (not swiglu) and bool(d.has_bias)
        return {
            "dx": (d.T, d.D), "dw_r": (d.D, d.M), "dw1": (d.M, n1, d.D), "dw2": (d.M, d.D, d.I),
            "db1": (d.M, d.I) if biases else None, "db2": (d.M, d.D) if biases else None,
            "dsh_w1": (2 * d.I_sh, d.D) if d.I_sh else None, "dsh_w2": (d.D, d.I_sh) if d.I_sh else None,
        }

    def backward(self, x: torch.Tensor, dy: torch.Tensor, grads: dict | None = None, stream=None) -> dict:
        """Gradients of L = sum(dy * MoE-FFN(x)) (moe_backward): dx in the
        layer's dtype, every parameter gradient in fp32.  The backward has its
        own workspace (allocated on first use); ``backward_view`` reads the
        routing it recomputed."""
        if self._bws is None:
            self.bws_bytes = abi.moe_backward_workspace_size(self.desc)
            if self.bws_bytes == 0:
                raise abi.MoEError("moe_backward_workspace_size", abi.MOE_ERR_INVALID_ARG)
            self._bws = torch.zeros(self.bws_bytes + 256, dtype=torch.uint8, device=self.device)
            self._bws_off = (-self._bws.data_ptr()) % 256
        if grads is None:
            grads = {}
            for name, shape in self.grad_shapes().items():
                if shape is not None:
                    dt = x.dtype if name == "dx" else torch.float32
                    grads[name] = torch.empty(shape, dtype=dt, device=self.device)
        g = abi.Grads()
        for name in abi.Grads._fields_:
            setattr(g, name[0], _ptr(grads.get(name[0])))
        abi.moe_backward(self.desc, self.weights, x.data_ptr(), dy.data_ptr(), g,
                         self._bws.data_ptr() + self._bws_off, self.bws_bytes, _stream_handle(stream))
        return grads

    def backward_status(self, stream=None) -> int:
        return abi.moe_device_status(self._bws.data_ptr() + self._bws_off, _stream_handle(stream))

    def backward_view(self, name: str) -> torch.Tensor:
        """The routing intermediate ``name`` of the last backward."""
        return self.view(name, ws=(self._bws, self._bws_off))

    def view(self, name: str, dtype=None, ws=None) -> torch.Tensor:
        """The intermediate ``name`` of the last forward, as a tensor view."""
        d = self.desc
        pairs = d.T * d.k
        shapes = {
            "status": ((1,), torch.int32), "topk_idx": ((d.T, d.k), torch.int32),
            "topk_w": ((d.T, d.k), torch.float32), "counts": ((d.M,), torch.int32),
            "offsets": ((d.M + 1,), torch.int32), "slot_of": ((d.T, d.k), torch.int32),
            "row_token": ((pairs,), torch.int32), "row_w": ((pairs,), torch.float32),
            "out_perm": ((pairs, d.D), torch.float32),
        }
        shape, dt = shapes[name]
        buf, base = (self.ws, self._ws_off) if ws is None else ws
        off = base + getattr(self.layout, name)
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty((), dtype=dt).element_size()
        return buf[off:off + nbytes].view(dt).view(*shape)


class DenseLayer:
    """One dense FFN layer (w1, b1, w2, b2 device tensors, kept alive here)."""

    def __init__(self, cfg: dict, tensors: dict, T: int | None = None):
        self.cfg = cfg
        self.tensors = tensors
        self.desc = dense_desc_from_config(cfg, T)
        for name in ("w1", "b1", "w2", "b2"):
            v = tensors.get(name)
            if v is not None and not v.is_contiguous():
                raise ValueError(f"{name} must be contiguous")
        self.ws_bytes = abi.moe_dense_ffn_workspace_size(self.desc)
        if self.ws_bytes == 0:
            raise abi.MoEError("moe_dense_ffn_workspace_size", abi.MOE_ERR_INVALID_ARG)
        self.ws = torch.zeros(self.ws_bytes + 256, dtype=torch.uint8, device=tensors["w1"].device)
        self._ws_off = (-self.ws.data_ptr()) % 256

    @property
    def ws_ptr(self) -> int:
        return self.ws.data_ptr() + self._ws_off

    def args(self):
        t = self.tensors
        return (_ptr(t["w1"]), _ptr(t.get("b1")), _ptr(t["w2"]), _ptr(t.get("b2")))

    def forward(self, x: torch.Tensor, addend: torch.Tensor | None = None, y: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
        """y = (addend +) FFN(x)."""
        if y is None:
            y = torch.empty_like(x)
        abi.moe_dense_ffn(self.desc, *self.args(), x.data_ptr(), _ptr(addend), y.data_ptr(), self.ws_ptr,
                          self.ws_bytes, _stream_handle(stream))
        return y

    def device_status(self, stream=None) -> int:
        return abi.moe_device_status(self.ws_ptr, _stream_handle(stream))

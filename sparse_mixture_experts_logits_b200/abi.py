"""ctypes binding of include/moe_b200.h (same names, same arguments).

Pointers are passed as Python ints (device addresses, e.g. tensor.data_ptr())
and the stream as an int (torch.cuda.Stream.cuda_stream) or None.  Every
wrapper raises MoEError when the library returns a status other than MOE_OK.
"""
from __future__ import annotations

import ctypes
import os

LIB_NAME = "libmoe_b200.so"
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), LIB_NAME)

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_DEVICE = range(5)
DTYPE_F32, DTYPE_BF16 = 0, 1
GATE_SOFTMAX, GATE_SIGMOID_BIAS = 0, 1
ACT_GELU_TANH, ACT_SWIGLU = 0, 1
DEVERR_NONE, DEVERR_BAD_EXPERT_INDEX, DEVERR_TIMEOUT, DEVERR_BAD_ROW_TOKEN, DEVERR_BAD_COUNT = 0, 1, 2, 3, 4

EXPORTED_SYMBOLS = [
    "moe_status_string", "moe_version", "moe_device_status",
    "moe_route_workspace_size", "moe_route_topk",
    "moe_permute_workspace_size", "moe_permute", "moe_permute_static_scratch",
    "moe_expert_ffn_workspace_size", "moe_expert_ffn",
    "moe_shared_expert_workspace_size", "moe_shared_expert",
    "moe_combine", "moe_workspace_size", "moe_workspace_layout", "moe_forward",
    "moe_forward_profiled", "moe_forward_launch_count", "moe_algorithmic_work",
    "moe_forward_add", "moe_dense_ffn_workspace_size", "moe_dense_ffn", "moe_dense_ffn_profiled",
    "moe_backward_workspace_size", "moe_backward", "moe_backward_launch_count", "moe_gather_rows",
    "moe_capacity_drop", "moe_expert_capacity", "moe_selftest_wait_timeout", "moe_ep_pack", "moe_ep_unpack",
]
NUM_STAGE_EVENTS = 9
NUM_DENSE_EVENTS = 3
STAGE_NAMES = ["route", "dispatch", "gather", "expert_up", "expert_down", "shared_up", "shared_down",
               "combine"]


class MoEError(RuntimeError):
    def __init__(self, func: str, status: int):
        self.status = status
        super().__init__(f"{func} failed: {_status_name(status)} ({status})")


class LayerDesc(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int), ("T", ctypes.c_int), ("D", ctypes.c_int), ("M", ctypes.c_int),
        ("k", ctypes.c_int), ("gate", ctypes.c_int), ("act", ctypes.c_int), ("I", ctypes.c_int),
        ("has_bias", ctypes.c_int), ("norm_topk_prob", ctypes.c_int),
        ("routed_scaling_factor", ctypes.c_float), ("eps", ctypes.c_float), ("I_sh", ctypes.c_int),
        ("n_group", ctypes.c_int), ("topk_group", ctypes.c_int),
    ]


class DenseDesc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("dtype", "T", "D", "I", "act", "has_bias")]


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w_r", "e_bias", "w1", "b1", "w2", "b2", "sh_w1", "sh_w2")]


class Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("dx", "dw_r", "dw1", "db1", "dw2", "db2", "dsh_w1", "dsh_w2")]


class WsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("status", "topk_idx", "topk_w", "counts", "offsets", "slot_of", "row_token",
                 "row_w", "out_perm", "total")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python sparse_mixture_experts_logits_b200/build.py` "
            "(there is no fallback path)")
    return ctypes.CDLL(LIB_PATH)


lib = _load()

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_P = ctypes.POINTER


def _decl(name, res, args):
    fn = getattr(lib, name)
    fn.restype = res
    fn.argtypes = args
    return fn


_decl("moe_status_string", ctypes.c_char_p, [_i])
_decl("moe_version", ctypes.c_char_p, [])
_decl("moe_device_status", _i, [_vp, _vp, _P(_i)])
_decl("moe_route_workspace_size", _sz, [_i, _i, _i, _i])
_decl("moe_route_topk", _i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _f, _i, _i, _vp, _vp, _vp, _sz,
                            _vp])
_decl("moe_permute_workspace_size", _sz, [_i, _i, _i])
_decl("moe_permute", _i, [_vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp])
_decl("moe_permute_static_scratch", _i, [_vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp])
_decl("moe_expert_ffn_workspace_size", _sz, [_P(LayerDesc)])
_decl("moe_expert_ffn", _i, [_P(LayerDesc), _P(Weights), _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp])
_decl("moe_shared_expert_workspace_size", _sz, [_P(LayerDesc)])
_decl("moe_shared_expert", _i, [_P(LayerDesc), _P(Weights), _vp, _vp, _vp, _sz, _vp])
_decl("moe_combine", _i, [_P(LayerDesc), _vp, _vp, _vp, _vp, _vp, _vp])
_decl("moe_workspace_size", _sz, [_P(LayerDesc)])
_decl("moe_workspace_layout", _i, [_P(LayerDesc), _P(WsLayout)])
_decl("moe_forward", _i, [_P(LayerDesc), _P(Weights), _vp, _vp, _vp, _sz, _vp])
_decl("moe_forward_profiled", _i, [_P(LayerDesc), _P(Weights), _vp, _vp, _vp, _sz, _vp, _P(_vp), _i])
_decl("moe_forward_launch_count", _i, [_P(LayerDesc)])
_decl("moe_algorithmic_work", None, [_P(LayerDesc), _vp, _P(ctypes.c_double), _P(ctypes.c_double)])
_decl("moe_forward_add", _i, [_P(LayerDesc), _P(Weights), _vp, _vp, _vp, _vp, _sz, _vp])
_decl("moe_dense_ffn_workspace_size", _sz, [_P(DenseDesc)])
_decl("moe_dense_ffn", _i, [_P(DenseDesc), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp])
_decl("moe_dense_ffn_profiled", _i, [_P(DenseDesc), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp,
                                     _P(_vp), _i])
_decl("moe_gather_rows", _i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp])
_decl("moe_capacity_drop", _i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp])
_decl("moe_ep_pack", _i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp])
_decl("moe_ep_unpack", _i, [_vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp])
_decl("moe_expert_capacity", _i, [ctypes.c_double, _i, _i, _i])
_decl("moe_selftest_wait_timeout", _i, [ctypes.c_uint64, _vp, _vp, _vp])
_decl("moe_backward_workspace_size", _sz, [_P(LayerDesc)])
_decl("moe_backward", _i, [_P(LayerDesc), _P(Weights), _vp, _vp, _P(Grads), _vp, _sz, _vp])
_decl("moe_backward_launch_count", _i, [_P(LayerDesc)])


def _status_name(s: int) -> str:
    return lib.moe_status_string(int(s)).decode()


def _check(func, status):
    if status != MOE_OK:
        raise MoEError(func, status)


def moe_status_string(s: int) -> str:
    return _status_name(s)


def moe_version() -> str:
    return lib.moe_version().decode()


def moe_device_status(ws: int, stream=None) -> int:
    out = ctypes.c_int(0)
    _check("moe_device_status", lib.moe_device_status(ws, stream, ctypes.byref(out)))
    return out.value


def moe_route_workspace_size(T, D, M, dtype) -> int:
    return lib.moe_route_workspace_size(T, D, M, dtype)


def moe_route_topk(x, w_r, e_bias, T, D, M, k, dtype, gate, norm_topk_prob, routed_scaling_factor,
                   eps, n_group, topk_group, topk_idx, topk_w, ws, ws_bytes, stream=None):
    _check("moe_route_topk", lib.moe_route_topk(
        x, w_r, e_bias, T, D, M, k, dtype, gate, norm_topk_prob, routed_scaling_factor, eps,
        n_group, topk_group, topk_idx, topk_w, ws, ws_bytes, stream))


def moe_permute_workspace_size(T, k, M) -> int:
    return lib.moe_permute_workspace_size(T, k, M)


def moe_permute(topk_idx, topk_w, T, k, M, counts, offsets, slot_of, row_token, row_w, ws, ws_bytes,
                stream=None):
    _check("moe_permute", lib.moe_permute(topk_idx, topk_w, T, k, M, counts, offsets, slot_of,
                                          row_token, row_w, ws, ws_bytes, stream))


def moe_permute_static_scratch(topk_idx, topk_w, T, k, M, counts, offsets, slot_of, row_token, row_w,
                               device_status=None, stream=None):
    """moe_permute without a workspace (scratch compiled into the library)."""
    _check("moe_permute_static_scratch", lib.moe_permute_static_scratch(
        topk_idx, topk_w, T, k, M, counts, offsets, slot_of, row_token, row_w, device_status, stream))


def moe_expert_ffn_workspace_size(desc: LayerDesc) -> int:
    return lib.moe_expert_ffn_workspace_size(ctypes.byref(desc))


def moe_expert_ffn(desc, weights, x, offsets, row_token, row_w, out_perm, ws, ws_bytes, stream=None):
    _check("moe_expert_ffn", lib.moe_expert_ffn(ctypes.byref(desc), ctypes.byref(weights), x, offsets,
                                                row_token, row_w, out_perm, ws, ws_bytes, stream))


def moe_shared_expert_workspace_size(desc: LayerDesc) -> int:
    return lib.moe_shared_expert_workspace_size(ctypes.byref(desc))


def moe_shared_expert(desc, weights, x, y_sh, ws, ws_bytes, stream=None):
    _check("moe_shared_expert", lib.moe_shared_expert(ctypes.byref(desc), ctypes.byref(weights), x,
                                                      y_sh, ws, ws_bytes, stream))


def moe_combine(desc, out_perm, slot_of, shared_out, addend, y, stream=None):
    _check("moe_combine", lib.moe_combine(ctypes.byref(desc), out_perm, slot_of, shared_out, addend, y,
                                          stream))


def moe_workspace_size(desc: LayerDesc) -> int:
    return lib.moe_workspace_size(ctypes.byref(desc))


def moe_workspace_layout(desc: LayerDesc) -> WsLayout:
    out = WsLayout()
    _check("moe_workspace_layout", lib.moe_workspace_layout(ctypes.byref(desc), ctypes.byref(out)))
    return out


def moe_forward(desc, weights, x, y, ws, ws_bytes, stream=None):
    _check("moe_forward", lib.moe_forward(ctypes.byref(desc), ctypes.byref(weights), x, y, ws, ws_bytes,
                                          stream))


def moe_forward_profiled(desc, weights, x, y, ws, ws_bytes, stream, events):
    """events: NUM_STAGE_EVENTS raw cudaEvent_t handles (ints)."""
    arr = (ctypes.c_void_p * len(events))(*events)
    _check("moe_forward_profiled", lib.moe_forward_profiled(
        ctypes.byref(desc), ctypes.byref(weights), x, y, ws, ws_bytes, stream, arr, len(events)))


def moe_forward_launch_count(desc) -> int:
    return lib.moe_forward_launch_count(ctypes.byref(desc))


def moe_algorithmic_work(desc: LayerDesc, counts_host=None):
    """(flops, bytes) of one forward given host int32 counts (a numpy array)."""
    f = ctypes.c_double(0.0)
    b = ctypes.c_double(0.0)
    ptr = None
    if counts_host is not None:
        import numpy as np
        counts_host = np.ascontiguousarray(counts_host, dtype=np.int32)
        ptr = counts_host.ctypes.data
    lib.moe_algorithmic_work(ctypes.byref(desc), ptr, ctypes.byref(f), ctypes.byref(b))
    return f.value, b.value


def moe_forward_add(desc, weights, x, addend, y, ws, ws_bytes, stream=None):
    _check("moe_forward_add", lib.moe_forward_add(ctypes.byref(desc), ctypes.byref(weights), x, addend, y,
                                                  ws, ws_bytes, stream))


def moe_dense_ffn_workspace_size(desc: DenseDesc) -> int:
    return lib.moe_dense_ffn_workspace_size(ctypes.byref(desc))


def moe_dense_ffn(desc, w1, b1, w2, b2, x, addend, y, ws, ws_bytes, stream=None):
    _check("moe_dense_ffn", lib.moe_dense_ffn(ctypes.byref(desc), w1, b1, w2, b2, x, addend, y, ws,
                                              ws_bytes, stream))


def moe_dense_ffn_profiled(desc, w1, b1, w2, b2, x, addend, y, ws, ws_bytes, stream, events):
    """events: NUM_DENSE_EVENTS raw cudaEvent_t handles (ints)."""
    arr = (ctypes.c_void_p * len(events))(*events)
    _check("moe_dense_ffn_profiled", lib.moe_dense_ffn_profiled(
        ctypes.byref(desc), w1, b1, w2, b2, x, addend, y, ws, ws_bytes, stream, arr, len(events)))


def moe_backward_workspace_size(desc: LayerDesc) -> int:
    return lib.moe_backward_workspace_size(ctypes.byref(desc))


def moe_backward(desc, weights, x, dy, grads, ws, ws_bytes, stream=None):
    _check("moe_backward", lib.moe_backward(ctypes.byref(desc), ctypes.byref(weights), x, dy,
                                            ctypes.byref(grads), ws, ws_bytes, stream))


def moe_backward_launch_count(desc) -> int:
    return lib.moe_backward_launch_count(ctypes.byref(desc))


def moe_gather_rows(x, row_token, n_rows, x_perm, rows, T, D, dtype, device_status=None, stream=None):
    _check("moe_gather_rows", lib.moe_gather_rows(x, row_token, n_rows, x_perm, rows, T, D, dtype, device_status,
                                                  stream))


def moe_capacity_drop(topk_idx, slot_of, offsets, T, k, M, capacity, stream=None):
    _check("moe_capacity_drop", lib.moe_capacity_drop(topk_idx, slot_of, offsets, T, k, M, capacity, stream))


def moe_ep_pack(x, offsets, row_token, row_w, slot_of, T, k, M, D, dtype, cap, x_pad, w_pad, slot_pad, kept,
                device_status=None, stream=None):
    _check("moe_ep_pack", lib.moe_ep_pack(x, offsets, row_token, row_w, slot_of, T, k, M, D, dtype, cap, x_pad,
                                          w_pad, slot_pad, kept, device_status, stream))


def moe_ep_unpack(recv_kept, w_recv, world, E, cap, offsets, row_token, row_w, slot_of, device_status=None,
                  stream=None):
    _check("moe_ep_unpack", lib.moe_ep_unpack(recv_kept, w_recv, world, E, cap, offsets, row_token, row_w,
                                              slot_of, device_status, stream))


def moe_expert_capacity(factor, T, k, M) -> int:
    return lib.moe_expert_capacity(float(factor), T, k, M)


def moe_selftest_wait_timeout(limit_ns, device_status, elapsed_ns=None, stream=None):
    _check("moe_selftest_wait_timeout",
           lib.moe_selftest_wait_timeout(int(limit_ns), device_status, elapsed_ns, stream))

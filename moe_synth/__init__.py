"""Seeded synthetic inputs for the sparse MoE FFN layer.

This module is the one place that both the CUDA path's tests/benchmark and
the CPU oracle take their inputs from.  It holds no arithmetic of the MoE
method itself: only a counter-based random generator and the shapes and
value distributions of the workloads.

Generator
---------
Every tensor is addressed by a string key (workload, tensor name, expert).
Element ``i`` of the flattened tensor is a pure function of (key, i):

    h(c)  = mix32(mix32(c XOR k1) XOR k2)          (c = 2*i and 2*i+1)
    u0..3 = the four 16-bit halves of h(2i), h(2i+1)
    s     = sum_j (2*u_j - 65535)                   (exact integer)
    value = s * (std / std_s)   in fp64, then rounded to fp32 (and bf16)

``mix32`` is the 32-bit integer finaliser x ^= x>>16; x *= 0x45d9f3b;
x ^= x>>16; x *= 0x45d9f3b; x ^= x>>16 (all mod 2^32), and (k1, k2) are
two 32-bit words of BLAKE2b(key).  ``s`` is an Irwin-Hall sum of four
uniforms, so values follow a normal law with the stated standard deviation,
truncated at +-3.46 sigma.  All steps are integer ops or correctly rounded
IEEE multiplies/conversions, so a tensor is bit-identical whether it is made
on the CPU or on a GPU, and any slice (a few rows of x, one expert's weights)
can be made without making the rest.
"""
from __future__ import annotations

import hashlib
import math

import torch

from .configs import CONFIGS, DENSE_CONFIGS, TEST_CONFIGS, get_config, all_config_names, dense_config_names  # noqa: F401,E501

_MASK32 = 0xFFFFFFFF
_MIX = 0x45D9F3B
# standard deviation of s = sum of four (2u - 65535), u uniform on 0..65535
_STD_S = math.sqrt(4.0 * (65536.0 ** 2 - 1.0) / 3.0)
_CHUNK = 1 << 24


def key_words(key: str) -> tuple[int, int]:
    d = hashlib.blake2b(key.encode("utf-8"), digest_size=8).digest()
    return int.from_bytes(d[:4], "little"), int.from_bytes(d[4:], "little")


def _mix32(x: torch.Tensor) -> torch.Tensor:
    # x holds values in [0, 2^32) in int64; products stay below 2^59
    x = ((x >> 16) ^ x) * _MIX & _MASK32
    x = ((x >> 16) ^ x) * _MIX & _MASK32
    return (x >> 16) ^ x


def _hash(counter: torch.Tensor, k1: int, k2: int) -> torch.Tensor:
    return _mix32(_mix32(counter ^ k1) ^ k2)


def _normal_from_index(idx: torch.Tensor, std: float, k1: int, k2: int) -> torch.Tensor:
    h0 = _hash(idx * 2, k1, k2)
    h1 = _hash(idx * 2 + 1, k1, k2)
    s = (2 * (h0 & 0xFFFF) - 65535) + (2 * (h0 >> 16) - 65535) \
        + (2 * (h1 & 0xFFFF) - 65535) + (2 * (h1 >> 16) - 65535)
    return (s.to(torch.float64) * (std / _STD_S)).to(torch.float32)


def _uniform_from_index(idx: torch.Tensor, lo: float, hi: float, k1: int, k2: int) -> torch.Tensor:
    h = _hash(idx, k1, k2)
    u = ((h >> 8).to(torch.float64) + 0.5) * (1.0 / (1 << 24))
    return (lo + (hi - lo) * u).to(torch.float32)


def normal(shape, std: float, key: str, device="cpu", dtype=torch.bfloat16,
           out: torch.Tensor | None = None) -> torch.Tensor:
    """Tensor of ``shape`` with N(0, std^2) entries (see module docstring)."""
    k1, k2 = key_words(key)
    n = int(math.prod(shape))
    if n >= (1 << 31):
        raise ValueError("tensor too large for one key; split it by expert")
    if out is None:
        out = torch.empty(n, dtype=dtype, device=device)
    flat = out.view(-1)
    for s0 in range(0, n, _CHUNK):
        s1 = min(n, s0 + _CHUNK)
        idx = torch.arange(s0, s1, dtype=torch.int64, device=flat.device)
        flat[s0:s1] = _normal_from_index(idx, std, k1, k2).to(dtype)
    return out.view(*shape)


def normal_rows(rows: torch.Tensor, ncols: int, std: float, key: str,
                dtype=torch.bfloat16) -> torch.Tensor:
    """Rows ``rows`` of the [*, ncols] tensor that ``normal`` makes for ``key``."""
    k1, k2 = key_words(key)
    rows = rows.to(torch.int64)
    idx = rows[:, None] * ncols + torch.arange(ncols, dtype=torch.int64, device=rows.device)[None, :]
    return _normal_from_index(idx.reshape(-1), std, k1, k2).to(dtype).view(rows.numel(), ncols)


def uniform(shape, lo: float, hi: float, key: str, device="cpu") -> torch.Tensor:
    k1, k2 = key_words(key)
    n = int(math.prod(shape))
    idx = torch.arange(n, dtype=torch.int64, device=device)
    return _uniform_from_index(idx, lo, hi, k1, k2).view(*shape)


def permutation(n: int, key: str) -> torch.Tensor:
    """Seeded permutation of 0..n-1 (argsort of hashed counters, CPU)."""
    k1, k2 = key_words(key)
    h = _hash(torch.arange(n, dtype=torch.int64), k1, k2)
    return torch.argsort(h * n + torch.arange(n, dtype=torch.int64))


# ---------------------------------------------------------------------------
# Layer inputs
# ---------------------------------------------------------------------------

def _key(cfg, *parts) -> str:
    return "/".join([cfg["name"], f"seed{cfg.get('seed', 0)}"] + [str(p) for p in parts])


def act_dtype(cfg):
    return torch.float32 if cfg["dtype"] == "f32" else torch.bfloat16


def expert_w1(cfg, e: int, device="cpu") -> torch.Tensor:
    """Expert e's input projection, nn.Linear layout [N1, D] (N1 = I or 2I)."""
    n1 = cfg["I"] * (2 if cfg["act"] == "swiglu" else 1)
    return normal((n1, cfg["D"]), 1.0 / math.sqrt(cfg["D"]), _key(cfg, "w1", e), device, act_dtype(cfg))


def expert_w2(cfg, e: int, device="cpu") -> torch.Tensor:
    """Expert e's output projection, nn.Linear layout [D, I]."""
    return normal((cfg["D"], cfg["I"]), 1.0 / math.sqrt(cfg["I"]), _key(cfg, "w2", e), device, act_dtype(cfg))


def expert_b1(cfg, e: int, device="cpu") -> torch.Tensor:
    return normal((cfg["I"],), cfg["bias_std"], _key(cfg, "b1", e), device, act_dtype(cfg))


def expert_b2(cfg, e: int, device="cpu") -> torch.Tensor:
    return normal((cfg["D"],), cfg["bias_std"], _key(cfg, "b2", e), device, act_dtype(cfg))


def x_tokens(cfg, device="cpu") -> torch.Tensor:
    return normal((cfg["T"], cfg["D"]), 1.0, _key(cfg, "x"), device, act_dtype(cfg))


def x_rows(cfg, rows: torch.Tensor) -> torch.Tensor:
    return normal_rows(rows, cfg["D"], 1.0, _key(cfg, "x"), act_dtype(cfg))


def router_weight(cfg, device="cpu") -> torch.Tensor:
    """W_r in the [D, M] layout."""
    return normal((cfg["D"], cfg["M"]), cfg["w_r_std"], _key(cfg, "w_r"), device, act_dtype(cfg))


def router_bias(cfg, device="cpu") -> torch.Tensor | None:
    """Correction bias e_bias[M] (fp32), or None for routers without one."""
    kind = cfg.get("e_bias")
    if kind is None:
        return None
    M = cfg["M"]
    if kind[0] == "uniform":
        return uniform((M,), kind[1], kind[2], _key(cfg, "e_bias"), device)
    if kind[0] == "zipf":
        # e_bias[pi(r)] = beta * log p_r with p_r proportional to r^-s, r = 1..M
        s, beta = kind[1], kind[2]
        r = torch.arange(1, M + 1, dtype=torch.float64)
        p = r ** (-s)
        p = p / p.sum()
        pi = permutation(M, _key(cfg, "zipf_perm"))
        out = torch.empty(M, dtype=torch.float64)
        out[pi] = beta * torch.log(p)
        return out.to(torch.float32).to(device)
    if kind[0] == "const":
        return torch.full((M,), float(kind[1]), dtype=torch.float32, device=device)
    raise ValueError(f"unknown e_bias kind {kind}")


def shared_w1(cfg, device="cpu") -> torch.Tensor | None:
    if not cfg.get("I_sh"):
        return None
    return normal((2 * cfg["I_sh"], cfg["D"]), 1.0 / math.sqrt(cfg["D"]), _key(cfg, "sh_w1"), device, act_dtype(cfg))


def shared_w2(cfg, device="cpu") -> torch.Tensor | None:
    if not cfg.get("I_sh"):
        return None
    return normal((cfg["D"], cfg["I_sh"]), 1.0 / math.sqrt(cfg["I_sh"]), _key(cfg, "sh_w2"), device, act_dtype(cfg))


def stacked(cfg, which: str, device="cpu") -> torch.Tensor | None:
    """All experts' ``which`` in one [M, ...] tensor (w1, w2, b1 or b2)."""
    fn = {"w1": expert_w1, "w2": expert_w2, "b1": expert_b1, "b2": expert_b2}[which]
    if which in ("b1", "b2") and not cfg.get("has_bias"):
        return None
    first = fn(cfg, 0, device)
    out = torch.empty((cfg["M"],) + tuple(first.shape), dtype=first.dtype, device=device)
    out[0] = first
    for e in range(1, cfg["M"]):
        out[e] = fn(cfg, e, device)
    return out


def layer_inputs(cfg, device="cpu") -> dict:
    """Every input of one layer call, as torch tensors on ``device``."""
    return {
        "x": x_tokens(cfg, device),
        "w_r": router_weight(cfg, device),
        "e_bias": router_bias(cfg, device),
        "w1": stacked(cfg, "w1", device),
        "b1": stacked(cfg, "b1", device),
        "w2": stacked(cfg, "w2", device),
        "b2": stacked(cfg, "b2", device),
        "sh_w1": shared_w1(cfg, device),
        "sh_w2": shared_w2(cfg, device),
    }


def addend_tokens(cfg, device="cpu") -> torch.Tensor:
    """The other term of a block sum (attention output or residual), [T, D]."""
    return normal((cfg["T"], cfg["D"]), 1.0, _key(cfg, "addend"), device, act_dtype(cfg))


def upstream_grad(cfg, device="cpu") -> torch.Tensor:
    """dL/dy of a backward pass, [T, D], N(0, 1) in the layer's dtype."""
    return normal((cfg["T"], cfg["D"]), 1.0, _key(cfg, "dy"), device, act_dtype(cfg))


def dense_inputs(cfg, device="cpu") -> dict:
    """Every input of one dense FFN layer call (the layer's weights are drawn
    like one expert's, under the name "dense")."""
    bias = bool(cfg.get("has_bias"))
    return {
        "x": x_tokens(cfg, device),
        "w1": expert_w1(cfg, "dense", device),
        "b1": expert_b1(cfg, "dense", device) if bias else None,
        "w2": expert_w2(cfg, "dense", device),
        "b2": expert_b2(cfg, "dense", device) if bias else None,
        "addend": addend_tokens(cfg, device),
    }

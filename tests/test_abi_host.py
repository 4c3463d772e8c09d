"""The C-ABI library loads and exports every symbol the header declares; the
host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

import moe_synth as ms

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def B():
    import __graft_entry__
    __graft_entry__._build_module().build()
    import sparse_mixture_experts_logits_b200 as B
    return B


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("moe_route_topk", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_forward"):
        assert required in names


def test_every_declared_symbol_is_exported(B):
    lib = ctypes.CDLL(B.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert sorted(B.EXPORTED_SYMBOLS) == declared_functions()


def test_version_and_status_strings(B):
    assert "sm_100a" in B.moe_version()
    assert B.moe_status_string(0) == "MOE_OK"
    assert B.moe_status_string(4) == "MOE_ERR_DEVICE"
    assert B.moe_status_string(99) == "MOE_ERR_UNKNOWN"


def test_struct_layout_matches_header(B):
    assert ctypes.sizeof(B.LayerDesc) == 15 * 4
    assert ctypes.sizeof(B.Weights) == 8 * 8
    assert ctypes.sizeof(B.WsLayout) == 10 * 8


def _desc(B, name, **kw):
    return B.desc_from_config(ms.get_config(name, **kw))


def test_invalid_arguments_are_rejected_on_the_host(B):
    d = _desc(B, "glm_small_bf16")
    w = B.Weights()
    # k > M, k < 1, bad dtype, bf16 width not a multiple of 16
    for field, value, code in [("k", 17, 1), ("k", 0, 1), ("dtype", 7, 2), ("D", 250, 2),
                               ("I", 100, 2), ("M", 2000, 2), ("act", 5, 1), ("T", -1, 1)]:
        dd = _desc(B, "glm_small_bf16")
        setattr(dd, field, value)
        with pytest.raises(B.MoEError) as e:
            B.moe_forward(dd, w, 1, 1, 256, 1 << 30)
        assert e.value.status == code, (field, value)
        assert B.moe_workspace_size(dd) == 0
    # null weights
    with pytest.raises(B.MoEError) as e:
        B.moe_forward(d, w, 1, 1, 256, 1 << 30)
    assert e.value.status == 1
    # workspace too small / misaligned
    w.w_r, w.w1, w.w2, w.sh_w1, w.sh_w2 = 256, 256, 256, 256, 256
    need = B.moe_workspace_size(d)
    with pytest.raises(B.MoEError) as e:
        B.moe_forward(d, w, 256, 256, 256, need - 1)
    assert e.value.status == 1
    with pytest.raises(B.MoEError) as e:
        B.moe_forward(d, w, 256, 256, 255, need)
    assert e.value.status == 1
    with pytest.raises(B.MoEError):
        B.moe_route_topk(256, 256, None, 10, 64, 8, 9, 1, 0, 1, 1.0, 1e-20, 1, 1, 256, 256, 256, 1 << 20)
    with pytest.raises(B.MoEError):
        B.moe_permute(256, 256, 10, 2, 8, 256, 256, 256, 256, 256, 256, 0)


@pytest.mark.parametrize("M,k,n_group,topk_group,status", [
    (8, 2, 3, 1, 1),     # M not a multiple of the group count
    (64, 2, 64, 4, 2),   # more than 32 groups
    (8, 2, 4, 0, 1),     # no group kept
    (8, 2, 4, 5, 1),     # more groups kept than exist
    (16, 5, 4, 1, 1),    # the kept groups hold fewer than k experts
])
def test_bad_group_limits_rejected_before_launch(B, M, k, n_group, topk_group, status):
    with pytest.raises(B.MoEError) as e:
        B.moe_route_topk(256, 256, None, 10, 64, M, k, 1, 1, 1, 1.0, 1e-20, n_group, topk_group,
                         256, 256, 256, 1 << 20)
    assert e.value.status == status
    d = _desc(B, "glm_small_bf16")
    d.M, d.k, d.n_group, d.topk_group = M, k, n_group, topk_group
    assert B.moe_workspace_size(d) == 0


def test_zero_tokens_launch_nothing(B):
    d = _desc(B, "glm_small_bf16", T=0)
    w = B.Weights()
    w.w_r, w.w1, w.w2, w.sh_w1, w.sh_w2 = 256, 256, 256, 256, 256
    B.moe_forward(d, w, None, None, None, 0)
    B.moe_route_topk(None, None, None, 0, 64, 8, 2, 1, 0, 1, 1.0, 1e-20, 1, 1, None, None, None, 0)
    B.moe_expert_ffn(d, w, None, None, None, None, None, None, 0)
    B.moe_combine(d, None, None, None, None, None)


def test_workspace_layout_is_aligned_and_ordered(B):
    for name in ms.all_config_names():
        d = _desc(B, name)
        L = B.moe_workspace_layout(d)
        offs = [L.status, L.topk_idx, L.topk_w, L.counts, L.offsets, L.slot_of, L.row_token,
                L.row_w, L.out_perm]
        assert all(o % 256 == 0 for o in offs)
        assert offs == sorted(offs) and L.total >= offs[-1] + d.T * d.k * d.D * (2 if d.dtype else 4)
        assert B.moe_workspace_size(d) == L.total
        assert B.moe_expert_ffn_workspace_size(d) > 0


def test_dense_workspace_and_bad_descs(B):
    for name in ms.dense_config_names():
        cfg = ms.get_config(name)
        d = B.dense_desc_from_config(cfg)
        es = 2 if cfg["dtype"] == "bf16" else 4
        assert B.moe_dense_ffn_workspace_size(d) >= cfg["T"] * cfg["I"] * es
    d = B.dense_desc_from_config(ms.get_config("glm_dense_small_bf16"))
    for field, value, status in [("D", 24, 2), ("I", 40, 2), ("act", 7, 1), ("dtype", 5, 2), ("T", -1, 1)]:
        bad = B.DenseDesc.from_buffer_copy(d)
        setattr(bad, field, value)
        assert B.moe_dense_ffn_workspace_size(bad) == 0
        with pytest.raises(B.MoEError) as e:
            B.moe_dense_ffn(bad, 256, None, 256, None, 256, None, 256, 256, 1 << 30)
        assert e.value.status == status
    # T = 0 launches nothing; missing weights are rejected before any launch
    zero = B.DenseDesc.from_buffer_copy(d)
    zero.T = 0
    B.moe_dense_ffn(zero, None, None, None, None, None, None, None, None, 0)
    with pytest.raises(B.MoEError):
        B.moe_dense_ffn(d, None, None, 256, None, 256, None, 256, 256, 1 << 30)


def test_algorithmic_work_closed_form(B):
    """FLOPs and bytes of the GLaM prefill layer from the shapes alone:
    every token runs 2 experts of 2*D*H*2 FLOPs; the router D*M*2 per token."""
    cfg = ms.get_config("glam_prefill_bf16")
    d = B.desc_from_config(cfg)
    T, D, M, H = cfg["T"], cfg["D"], cfg["M"], cfg["I"]
    counts = np.full(M, T * 2 // M, dtype=np.int32)
    f, b = B.moe_algorithmic_work(d, counts)
    assert f == 2 * T * D * M + T * 2 * (2 * D * H * 2)
    weights = M * (2 * D * H + H + D) * 2
    assert b == weights + D * M * 2 + 2 * T * D * 2
    assert abs(f / 1e12 - 1.1017) < 1e-3
    # untouched experts cost no bytes
    counts[1:] = 0
    counts[0] = T * 2
    f2, b2 = B.moe_algorithmic_work(d, counts)
    assert f2 == f and b2 == (2 * D * H + H + D) * 2 + D * M * 2 + 2 * T * D * 2
    # GLM-5 shared expert bytes: 3 * 6144 * 2048 parameters at 2 bytes
    cfg5 = ms.get_config("glm5_skewed_prefill_bf16")
    d5 = B.desc_from_config(cfg5)
    f5, b5 = B.moe_algorithmic_work(d5, np.zeros(cfg5["M"], np.int32))
    assert b5 == 37748736 * 2 + 6144 * 256 * 2 + 4 * 256 + 2 * cfg5["T"] * 6144 * 2


def test_backward_host_checks(B):
    """moe_backward validates its descriptor and every required gradient
    pointer before touching the device."""
    for name in ms.all_config_names():
        d = _desc(B, name)
        assert B.moe_backward_workspace_size(d) > B.moe_workspace_size(d)
        assert B.moe_backward_launch_count(d) > B.moe_forward_launch_count(d)
    d = _desc(B, "glm_small_bf16")
    w = B.Weights()
    w.w_r, w.w1, w.w2, w.sh_w1, w.sh_w2 = 256, 256, 256, 256, 256
    full = dict(dx=256, dw_r=256, dw1=256, dw2=256, dsh_w1=256, dsh_w2=256)
    need = B.moe_backward_workspace_size(d)
    for missing in ("dw_r", "dw1", "dw2", "dsh_w1", "dsh_w2"):
        g = B.Grads(**{k: v for k, v in full.items() if k != missing})
        with pytest.raises(B.MoEError) as e:
            B.moe_backward(d, w, 256, 256, g, 256, need)
        assert e.value.status == 1, missing
    g = B.Grads(**full)
    with pytest.raises(B.MoEError) as e:     # workspace one byte short
        B.moe_backward(d, w, 256, 256, g, 256, need - 1)
    assert e.value.status == 1
    # GELU with biases needs db1 and db2
    dg = _desc(B, "glam_small_bf16")
    wg = B.Weights()
    wg.w_r, wg.w1, wg.w2, wg.b1, wg.b2 = 256, 256, 256, 256, 256
    with pytest.raises(B.MoEError) as e:
        B.moe_backward(dg, wg, 256, 256, B.Grads(dx=256, dw_r=256, dw1=256, dw2=256, db1=256), 256,
                       B.moe_backward_workspace_size(dg))
    assert e.value.status == 1
    bad = _desc(B, "glm_small_bf16")
    bad.k = 0
    assert B.moe_backward_workspace_size(bad) == 0 and B.moe_backward_launch_count(bad) == 0


def test_bf16_tma_operands_must_be_16_byte_aligned(B):
    """bf16 tensors the TMA kernels read, and the fp32 weight gradients they
    write, are checked for 16-byte alignment before any launch."""
    d = _desc(B, "glm_small_bf16")
    need = B.moe_backward_workspace_size(d)
    full = dict(dx=256, dw_r=256, dw1=256, dw2=256, dsh_w1=256, dsh_w2=256)
    for field in ("w_r", "w1", "w2", "sh_w1", "sh_w2"):
        w = B.Weights()
        w.w_r, w.w1, w.w2, w.sh_w1, w.sh_w2 = 256, 256, 256, 256, 256
        setattr(w, field, 264)
        with pytest.raises(B.MoEError) as e:
            B.moe_forward(d, w, 256, 256, 256, B.moe_workspace_size(d))
        assert e.value.status == 1, field
        with pytest.raises(B.MoEError) as e:
            B.moe_backward(d, w, 256, 256, B.Grads(**full), 256, need)
        assert e.value.status == 1, field
    w = B.Weights()
    w.w_r, w.w1, w.w2, w.sh_w1, w.sh_w2 = 256, 256, 256, 256, 256
    for x, dy in ((258, 256), (256, 260)):
        with pytest.raises(B.MoEError) as e:
            B.moe_backward(d, w, x, dy, B.Grads(**full), 256, need)
        assert e.value.status == 1
    with pytest.raises(B.MoEError) as e:
        B.moe_forward(d, w, 258, 256, 256, B.moe_workspace_size(d))
    assert e.value.status == 1
    for field in ("dw1", "dw2", "dsh_w1", "dsh_w2"):
        g = B.Grads(**dict(full, **{field: 260}))
        with pytest.raises(B.MoEError) as e:
            B.moe_backward(d, w, 256, 256, g, 256, need)
        assert e.value.status == 1, field


def test_gather_rows_host_checks(B):
    with pytest.raises(B.MoEError) as e:
        B.moe_gather_rows(256, 256, None, 256, -1, 4, 8, 1)
    assert e.value.status == 1
    with pytest.raises(B.MoEError) as e:
        B.moe_gather_rows(256, 256, None, 256, 4, 4, 8, 7)
    assert e.value.status == 2
    with pytest.raises(B.MoEError) as e:
        B.moe_gather_rows(None, 256, None, 256, 4, 4, 8, 1)
    assert e.value.status == 1
    B.moe_gather_rows(None, None, None, None, 0, 4, 8, 1)   # zero rows: nothing to do


def test_capacity_host_checks(B):
    import oracle
    for factor, T, k, M in ((1.0, 8192, 2, 64), (1.25, 300, 4, 16), (0.5, 333, 2, 8), (0.0, 10, 2, 4),
                            (2.0, 1, 8, 160), (1.0, 0, 2, 8)):
        assert B.moe_expert_capacity(factor, T, k, M) == oracle.expert_capacity(factor, T, k, M)
    assert B.moe_expert_capacity(-1.0, 10, 2, 4) == -1 and B.moe_expert_capacity(1.0, 10, 2, 0) == -1
    for args, status in [((256, 256, 256, 10, 2, 8, -1), 1), ((256, 256, 256, 10, 0, 8, 4), 1),
                         ((None, 256, 256, 10, 2, 8, 4), 1), ((256, 256, 256, 10, 2, 2000, 4), 2)]:
        with pytest.raises(B.MoEError) as e:
            B.moe_capacity_drop(*args)
        assert e.value.status == status
    B.moe_capacity_drop(None, None, None, 0, 2, 8, 4)   # T = 0: nothing to do


def _header_signatures():
    """name -> list of parameter declarations, from include/moe_b200.h."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    sigs = {}
    for m in re.finditer(r"\b(moe_[a-z_0-9]+)\s*\(([^;{]*?)\)\s*;", src, flags=re.S):
        params = " ".join(m.group(2).split())
        sigs[m.group(1)] = [] if params in ("", "void") else [p.strip() for p in params.split(",")]
    return sigs


def test_binding_arity_and_kinds_match_the_header(B):
    """ctypes does not check a call against the C declaration: every
    binding's argtypes must have the header's parameter count, with pointers
    where the header has pointers and numbers where it has numbers."""
    import ctypes
    sigs = _header_signatures()
    assert set(sigs) == set(B.EXPORTED_SYMBOLS)
    lib = B.lib
    for name, params in sigs.items():
        argtypes = getattr(lib, name).argtypes
        assert argtypes is not None, name
        assert len(argtypes) == len(params), (name, len(argtypes), params)
        for p, a in zip(params, argtypes):
            is_ptr = "*" in p
            ptr_like = a is ctypes.c_void_p or a is ctypes.c_char_p or hasattr(a, "_type_") and \
                isinstance(a, type(ctypes.POINTER(ctypes.c_int)))
            assert is_ptr == bool(ptr_like), (name, p, a)
            if not is_ptr:
                ctype = p.split()[0]
                expect = {"int": ctypes.c_int, "float": ctypes.c_float, "double": ctypes.c_double,
                          "size_t": ctypes.c_size_t, "moe_status_t": ctypes.c_int,
                          "uint64_t": ctypes.c_uint64}[ctype]
                assert a is expect, (name, p, a)


def test_struct_fields_match_the_header(B):
    """Every ctypes struct lists the header struct's fields, in order, with
    the header's types (int, float, size_t, pointer)."""
    import ctypes
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    structs = {}
    for m in re.finditer(r"typedef struct \{(.*?)\}\s*(moe_[a-z_]+_t)\s*;", src, flags=re.S):
        fields = []
        for decl in m.group(1).split(";"):
            decl = " ".join(decl.split())
            if not decl:
                continue
            for name in decl.split(",") if "*" not in decl else [decl]:
                fields.append(name)
        structs[m.group(2)] = fields
    pairs = {"moe_layer_desc_t": B.LayerDesc, "moe_weights_t": B.Weights, "moe_ws_layout_t": B.WsLayout,
             "moe_dense_desc_t": B.DenseDesc, "moe_grads_t": B.Grads}
    assert set(pairs) == set(structs)
    for cname, cls in pairs.items():
        expanded = []
        for decl in structs[cname]:
            parts = decl.replace("*", " * ").split()
            if "*" in parts:
                expanded.append((parts[-1], "ptr"))
            else:
                ctype = parts[0]
                for i, tok in enumerate(parts[1:]):
                    expanded.append((tok.strip(), ctype))
        names = [f[0] for f in cls._fields_]
        assert names == [n for n, _ in expanded], (cname, names, expanded)
        kinds = {"int": ctypes.c_int, "float": ctypes.c_float, "size_t": ctypes.c_size_t, "ptr": ctypes.c_void_p}
        for (n, t), (fname, ftype) in zip(expanded, cls._fields_):
            assert ftype is kinds[t], (cname, n, t, ftype)


def test_constants_match_the_header(B):
    """Status codes, enum values, device error codes and event counts of the
    binding equal the header's."""
    from sparse_mixture_experts_logits_b200 import abi
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    values = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(MOE_[A-Z_0-9]+)\s*=\s*(\d+)", src)}
    values.update({m.group(1): int(m.group(2)) for m in re.finditer(r"#define (MOE_[A-Z_0-9]+) (\d+)", src)})
    assert len(values) >= 17
    for name, v in values.items():
        attr = name if name.startswith(("MOE_OK", "MOE_ERR_")) else name[len("MOE_"):]
        assert getattr(abi, attr) == v, (name, v)

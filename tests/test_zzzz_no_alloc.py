"""moe_permute_static_scratch: the dispatch for callers that cannot allocate
device memory (their memory is owned by a pool, or the routing sits in a
loop that cannot take cudaMalloc's synchronisation, or a plug-in host gives
them no allocator).  It keeps its scratch in an array compiled into the
library, so it must give exactly what moe_permute gives with a workspace,
and a second call must not be disturbed by what the first left behind.

This file is collected last on purpose (test_zzzz_*), so that a run stopping
at the first failure has already run every other test."""
import numpy as np
import pytest
import torch

import moe_synth as ms

pytestmark = pytest.mark.gpu


def _permute_both(B, idx, w, M):
    T, k = idx.shape
    dev = idx.device
    s = torch.cuda.current_stream().cuda_stream

    def outs():
        return [torch.full((M,), -7, dtype=torch.int32, device=dev),
                torch.full((M + 1,), -7, dtype=torch.int32, device=dev),
                torch.full((T, k), -7, dtype=torch.int32, device=dev),
                torch.full((T * k,), -7, dtype=torch.int32, device=dev),
                torch.full((T * k,), -7.0, dtype=torch.float32, device=dev)]

    ref = outs()
    nbytes = B.moe_permute_workspace_size(T, k, M)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    B.moe_permute(idx.data_ptr(), w.data_ptr(), T, k, M, *[o.data_ptr() for o in ref], ws.data_ptr(),
                  nbytes, s)
    got = outs()
    status = torch.full((1,), 5, dtype=torch.int32, device=dev)
    B.moe_permute_static_scratch(idx.data_ptr(), w.data_ptr(), T, k, M, *[o.data_ptr() for o in got],
                                 status.data_ptr(), s)
    torch.cuda.synchronize()
    return ref, got, int(status.item())


def test_static_scratch_permute_matches_workspace_permute_twice():
    import sparse_mixture_experts_logits_b200 as B
    dev = "cuda"
    # call 1: a full-size routing (GLM-4.5 prefill shapes, 131072 pairs, 160 experts)
    cfg = ms.get_config("glm45_prefill_bf16")
    g = torch.Generator(device="cpu").manual_seed(0)
    T, k, M = cfg["T"], cfg["k"], cfg["M"]
    idx1 = torch.stack([torch.randperm(M, generator=g)[:k] for _ in range(T)]).to(torch.int32).to(dev)
    w1 = torch.rand(T, k, generator=g).to(dev)
    # call 2, right after: a smaller, skewed routing with empty experts, so
    # that stale scratch from call 1 would show up if it leaked through
    T2, k2, M2 = 777, 4, 48
    idx2 = torch.stack([torch.randperm(6, generator=g)[:k2] * 7 for _ in range(T2)]).to(torch.int32).to(dev)
    w2 = torch.rand(T2, k2, generator=g).to(dev)
    for idx, w, m in [(idx1, w1, M), (idx2, w2, M2)]:
        ref, got, status = _permute_both(B, idx, w, m)
        assert status == 0
        for a, b in zip(ref, got):
            assert torch.equal(a.view(torch.int32), b.view(torch.int32))
        assert int(got[1][-1]) == idx.numel()

    # the call itself takes no device memory: free memory is unchanged across
    # a further call (the outputs are allocated before the first reading)
    outs = [torch.empty(n, dtype=dt, device=dev) for n, dt in
            [(M, torch.int32), (M + 1, torch.int32), (T * k, torch.int32), (T * k, torch.int32),
             (T * k, torch.float32)]]
    s = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    B.moe_permute_static_scratch(idx1.data_ptr(), w1.data_ptr(), T, k, M, *[o.data_ptr() for o in outs], None, s)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before


def test_static_scratch_limits_and_errors():
    import sparse_mixture_experts_logits_b200 as B
    # beyond the compiled-in scratch: rejected on the host, nothing launched
    with pytest.raises(B.MoEError) as e:
        B.moe_permute_static_scratch(256, 256, 1 << 20, 8, 1024, 256, 256, 256, 256, 256, None, None)
    assert e.value.status == 2
    with pytest.raises(B.MoEError) as e:
        B.moe_permute_static_scratch(256, 256, 10, 9, 8, 256, 256, 256, 256, 256, None, None)
    assert e.value.status == 1
    # an out-of-range expert index is reported through the caller's status word
    dev = "cuda"
    idx = torch.randint(0, 8, (50, 2), dtype=torch.int32, device=dev)
    idx[7, 1] = 99
    w = torch.rand(50, 2, device=dev)
    outs = [torch.empty(n, dtype=dt, device=dev) for n, dt in
            [(8, torch.int32), (9, torch.int32), (100, torch.int32), (100, torch.int32), (100, torch.float32)]]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    B.moe_permute_static_scratch(idx.data_ptr(), w.data_ptr(), 50, 2, 8, *[o.data_ptr() for o in outs],
                                 status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert int(status.item()) == B.DEVERR_BAD_EXPERT_INDEX
    assert int(outs[0].sum()) == 99

"""The expiry branch of the library's bounded waits, exercised on a GPU in
the allowed form: a kernel waits on a barrier that nothing arrives on, with a
short limit.  It must give up on time, report MOE_DEVERR_TIMEOUT, make the
kernel's other waiter leave on the abort flag, and leave the context usable:
a whole layer run right after it still matches the oracle."""
import pytest
import torch

import moe_synth as ms
from test_gpu_parity import check_layer

pytestmark = pytest.mark.gpu

LIMIT_NS = 1_000_000  # 1 ms


def test_wait_gives_up_and_context_survives():
    import sparse_mixture_experts_logits_b200 as B
    dev = "cuda"
    status = torch.full((1,), 7, dtype=torch.int32, device=dev)
    elapsed = torch.zeros(2, dtype=torch.int64, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    B.moe_selftest_wait_timeout(LIMIT_NS, status.data_ptr(), elapsed.data_ptr(), s)
    torch.cuda.synchronize()
    assert int(status.item()) == B.DEVERR_TIMEOUT
    e = [int(v) for v in elapsed.cpu()]
    assert all(v >= 0 for v in e), "a wait returned success on a barrier nothing arrived on"
    # warp 0 gave up after its limit (and not absurdly later) ...
    assert LIMIT_NS <= e[0] < 200 * LIMIT_NS, e
    # ... and warp 1 left on the abort flag, before its own limit of 4 ms
    assert e[1] < 4 * LIMIT_NS, e
    # out-of-range limits are refused on the host
    with pytest.raises(B.MoEError):
        B.moe_selftest_wait_timeout(10, status.data_ptr(), None, s)
    # the context still works: a whole layer, checked against the oracle
    check_layer(B, ms.get_config("glm_small_bf16"), all_tokens=True)

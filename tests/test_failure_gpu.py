"""Failure detection without a GPU fault: a bounded in-kernel wait runs out on
a barrier nothing completes, the kernel records ATTN_ERR_TIMEOUT and returns,
and the context stays usable for the next launch."""
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import exact_attention_ring_b200 as eab  # noqa: E402

ATTN_OK, ATTN_ERR_TIMEOUT = 0, 4


def test_bounded_wait_times_out_and_context_survives():
    assert eab.attn_device_status() == ATTN_OK
    eab.attn_selftest_bounded_wait(20_000)  # 20 ms
    assert eab.attn_device_status() == ATTN_ERR_TIMEOUT
    assert eab.attn_device_status() == ATTN_OK  # reading clears it
    q = torch.randn(1, 2, 130, 64, device="cuda").to(torch.bfloat16)
    o, lse = eab.attention(q, q[:, :1].contiguous(), q[:, :1].contiguous(), causal=True)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and eab.attn_device_status() == ATTN_OK

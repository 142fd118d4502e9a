"""GPU parity of the fp16 calls (attn_fwd_f16, attn_decode_splitkv_f16,
attn_combine_f16) against the float64 oracle on fp16 inputs: same shapes,
tolerances and bit-exact structure checks as the bf16 path."""
import pytest
import torch

import oracle
import seeded_inputs as si
from attn_check import assert_attn_close

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import exact_attention_ring_b200 as eab  # noqa: E402  (must load: no fallback)

DEV = "cuda"
F16 = torch.float16


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,Hq,Hkv,N", [(1, 2, 2, 1), (1, 4, 2, 300), (2, 4, 1, 640), (1, 2, 2, 1000)])
def test_fwd_f16_matches_oracle(B, Hq, Hkv, N, d, causal):
    q, k, v = si.make_qkv(700 + N, B, Hq, Hkv, N, d, dtype=F16)
    o, lse = eab.attention(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=d ** -0.5)
    torch.cuda.synchronize()
    assert o.dtype == F16 and eab.attn_device_status() == 0
    o_ref, lse_ref = oracle.attention(q, k, v, causal, d ** -0.5)
    assert_attn_close(o, lse, o_ref, lse_ref, f"fp16 B{B} Hq{Hq} Hkv{Hkv} N{N} d{d} causal={causal}")


@pytest.mark.parametrize("d", [64, 128])
def test_fwd_f16_split_last_round(d):
    """fp16 through the two launches of a non-causal call whose last round is
    split (B1 Hq32 Hkv8 N1536: 192 query blocks, 44 of them split on 148 SMs)."""
    B, Hq, Hkv, N = 1, 32, 8, 1536
    q, k, v = si.make_qkv(760 + d, B, Hq, Hkv, N, d, dtype=F16)
    o, lse = eab.attention(q.to(DEV), k.to(DEV), v.to(DEV), causal=False, scale=d ** -0.5)
    torch.cuda.synchronize()
    assert o.dtype == F16 and eab.attn_device_status() == 0
    o_ref, lse_ref = oracle.attention(q, k, v, False, d ** -0.5)
    assert_attn_close(o, lse, o_ref, lse_ref, f"fp16 split B{B} Hq{Hq} Hkv{Hkv} N{N} d{d}")


def test_fwd_f16_large_logits_sampled():
    """LLaMA-7B shape with Q x 8 (exact in fp16) on sampled rows."""
    B, H, N, d = 2, 32, 2048, 128
    q, k, v = si.make_qkv(1001, B, H, H, N, d, 8.0, dtype=F16)
    for causal in (False, True):
        o, lse = eab.attention(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=d ** -0.5)
        torch.cuda.synchronize()
        rows = si.sample_rows(8, B, H, N, per_slice=64, max_slices=4)
        o_ref, lse_ref = oracle.attention(q, k, v, causal, d ** -0.5, rows=rows)
        assert_attn_close(o.reshape(-1, d)[rows.to(DEV)], lse.reshape(-1)[rows.to(DEV)], o_ref, lse_ref,
                          f"fp16 Qx8 causal={causal}")


def test_fwd_f16_causal_row0_is_v0_exactly():
    """Row 0 sees key 0 only: p = exp2(0) = 1, so O = V[0] bit for bit."""
    q, k, v = si.make_qkv(9, 1, 4, 2, 200, 128, dtype=F16)
    o, _ = eab.attention(q.to(DEV), k.to(DEV), v.to(DEV), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o[:, :, 0].cpu(), v.repeat_interleave(2, dim=1)[:, :, 0])


@pytest.mark.parametrize("B,Hq,Hkv,L,d", [(1, 32, 8, 4096, 128), (2, 8, 8, 1000, 128), (2, 4, 1, 777, 64),
                                          (1, 32, 8, 32768, 128)])
def test_decode_f16_matches_oracle(B, Hq, Hkv, L, d):
    q, k, v = si.make_decode(900 + L, B, Hq, Hkv, L, d, dtype=F16)
    o, lse = eab.decode(q.to(DEV), k.to(DEV), v.to(DEV), d ** -0.5)
    torch.cuda.synchronize()
    assert o.dtype == F16 and eab.attn_device_status() == 0
    o_ref, lse_ref = oracle.decode(q, k, v, d ** -0.5)
    assert_attn_close(o, lse, o_ref, lse_ref, f"fp16 decode B{B} Hq{Hq} Hkv{Hkv} L{L} d{d}")

"""GPU parity of split-KV decode and the combine against the float64 oracle."""
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


def gpu_partials(q, k, v, S, scale):
    B, Hq, d = q.shape
    o_part = torch.empty(B, Hq, S, d, device=DEV)
    lse_part = torch.empty(B, Hq, S, device=DEV)
    eab.attn_decode_splitkv(q.to(DEV), k.to(DEV), v.to(DEV), o_part, lse_part, S, scale)
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    return o_part, lse_part


def gpu_combine(o_part, lse_part):
    B, Hq, S, d = o_part.shape
    o = torch.empty(B, Hq, d, device=DEV, dtype=torch.bfloat16)
    lse = torch.empty(B, Hq, device=DEV)
    eab.attn_combine(o_part, lse_part, o, lse)
    torch.cuda.synchronize()
    return o, lse


@pytest.mark.parametrize("B,Hq,Hkv,L,d", [(1, 32, 8, 4096, 128), (2, 8, 8, 1000, 128), (2, 4, 1, 777, 64),
                                          (1, 6, 2, 300, 128), (1, 3, 1, 513, 64), (3, 16, 2, 2049, 128),
                                          (1, 2, 2, 1, 128), (1, 4, 4, 31, 64), (1, 24, 1, 1500, 128),
                                          (2, 40, 2, 900, 128), (1, 32, 1, 1000, 128), (1, 64, 1, 700, 128)])
def test_decode_full(B, Hq, Hkv, L, d):
    """Group sizes G = Hq / Hkv from 1 to 64: up to 32 at d = 128 the kernel with the
    keys as tile rows (16 or 32 query columns), otherwise the query heads as rows."""
    q, k, v = si.make_decode(5000 + L, B, Hq, Hkv, L, d)
    S = eab.attn_decode_default_splits(B, Hq, Hkv, L)
    chunk = eab.decode_chunk(L, S)
    op, lp = gpu_partials(q, k, v, S, d ** -0.5)
    # partials against the oracle's partials for the same key ranges
    op_ref, lp_ref = oracle.decode_partials(q, k, v, d ** -0.5, S, chunk)
    nonempty = torch.isfinite(lp_ref)
    assert torch.equal(torch.isfinite(lp.cpu()), nonempty)
    assert torch.all(op.cpu()[~nonempty] == 0)
    assert_attn_close(op.cpu()[nonempty], lp.cpu()[nonempty], op_ref[nonempty], lp_ref[nonempty], "partials")
    o, lse = gpu_combine(op, lp)
    o_ref, lse_ref = oracle.decode(q, k, v, d ** -0.5)
    assert_attn_close(o, lse, o_ref, lse_ref, f"decode B{B} Hq{Hq} Hkv{Hkv} L{L} d{d}")


@pytest.mark.parametrize("S", [1, 2, 7, 33, 64, 100])
def test_split_count_sweep(S):
    """Any split count, including ones that leave trailing splits empty."""
    B, Hq, Hkv, L, d = 1, 8, 2, 100, 128
    q, k, v = si.make_decode(5100, B, Hq, Hkv, L, d)
    op, lp = gpu_partials(q, k, v, S, d ** -0.5)
    o, lse = gpu_combine(op, lp)
    o_ref, lse_ref = oracle.decode(q, k, v, d ** -0.5)
    assert_attn_close(o, lse, o_ref, lse_ref, f"S={S}")


@pytest.mark.parametrize("G", [4, 24])
def test_decode_large_logits(G):
    """Q x 8 (exact in bf16): the running maximum of a query column jumps between
    key tiles, so the lazy rescale of O runs; partials and the merge against the oracle."""
    B, Hkv, L, d = 1, 2, 3000, 128
    q, k, v = si.make_decode(5150 + G, B, G * Hkv, Hkv, L, d)
    q = (q.float() * 8).to(torch.bfloat16)
    S = 5
    chunk = eab.decode_chunk(L, S)
    op, lp = gpu_partials(q, k, v, S, d ** -0.5)
    op_ref, lp_ref = oracle.decode_partials(q, k, v, d ** -0.5, S, chunk)
    assert_attn_close(op.cpu(), lp.cpu(), op_ref, lp_ref, f"partials Qx8 G{G}")
    o, lse = gpu_combine(op, lp)
    o_ref, lse_ref = oracle.decode(q, k, v, d ** -0.5)
    assert_attn_close(o, lse, o_ref, lse_ref, f"decode Qx8 G{G}")


def test_combine_alone():
    """attn_combine against the oracle's merge of the very same partials."""
    B, Hq, Hkv, L, d = 2, 8, 4, 5000, 128
    q, k, v = si.make_decode(5200, B, Hq, Hkv, L, d)
    op, lp = gpu_partials(q, k, v, 40, d ** -0.5)
    o, lse = gpu_combine(op, lp)
    o_ref, lse_ref = oracle.combine(op.cpu().double(), lp.cpu().double())
    assert_attn_close(o, lse, o_ref, lse_ref, "combine")


def test_combine_hand_partials():
    """Weights follow the LSEs: a -inf split is ignored, equal LSEs average."""
    o_part = torch.zeros(1, 1, 3, 64, device=DEV)
    o_part[0, 0, 0] = 1.0
    o_part[0, 0, 1] = 3.0
    o_part[0, 0, 2] = 1000.0
    lse_part = torch.tensor([[[0.5, 0.5, float("-inf")]]], device=DEV)
    o, lse = gpu_combine(o_part, lse_part)
    assert torch.all(o.float() == 2.0)
    assert abs(lse.item() - (0.5 + torch.log(torch.tensor(2.0)).item())) < 1e-6


def test_decode_equals_last_prefill_row():
    """Decode of query L-1 over L keys = row L-1 of causal prefill."""
    B, H, L, d = 1, 4, 700, 128
    q, k, v = si.make_qkv(5300, B, H, H, L, d)
    o_pre, lse_pre = eab.attention(q.to(DEV), k.to(DEV), v.to(DEV), causal=True)
    o_dec, lse_dec = eab.decode(q[:, :, L - 1].contiguous().to(DEV), k.to(DEV), v.to(DEV))
    torch.cuda.synchronize()
    assert (o_pre[:, :, L - 1].float() - o_dec.float()).abs().max().item() <= 2e-2
    assert (lse_pre[:, :, L - 1] - lse_dec).abs().max().item() <= 1e-3


@pytest.mark.parametrize("shape", si.DECODE, ids=[s.name for s in si.DECODE])
def test_decode_configs(shape):
    """The flash-decoding workloads at full size, in the bench's launch configuration
    (default split count); the oracle checks a sample of (batch, head) rows."""
    q, k, v = si.make_decode(shape.seed, shape.B, shape.Hq, shape.Hkv, shape.L, shape.d)
    o, lse = eab.decode(q.to(DEV), k.to(DEV), v.to(DEV), shape.scale)
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    n = shape.B * shape.Hq
    gen = torch.Generator().manual_seed(shape.seed + 1)
    rows = torch.randperm(n, generator=gen)[: min(n, 24)].sort().values
    o_ref, lse_ref = oracle.decode(q, k, v, shape.scale, rows=rows)
    assert_attn_close(o.reshape(n, -1)[rows.to(DEV)], lse.reshape(n)[rows.to(DEV)], o_ref, lse_ref, shape.name)

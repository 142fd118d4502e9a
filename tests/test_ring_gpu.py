"""GPU parity of ring attention (context parallelism) against the float64 oracle.

attn_fwd_f32 is attn_fwd before the rounding of O to bf16; attn_merge is
checked against the oracle's log-sum-exp merge of the same two partials; the
ring's per-rank steps (attn_fwd_f32 per key/value shard, attn_merge)
run for P virtual ranks on this one GPU (ring_attention_emulated) and must
reproduce exact attention over the whole sequence. A ring of one rank is
attn_fwd itself, bit for bit.
"""
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


def _partials(seed, rows, d):
    g = torch.Generator().manual_seed(seed)
    o_acc = torch.randn(rows, d, generator=g)
    o_blk = torch.randn(rows, d, generator=g)
    lse_acc = torch.randn(rows, generator=g) * 4.0
    lse_blk = torch.randn(rows, generator=g) * 4.0
    # rows where one side dominates by far, and rows where one side is empty
    lse_blk[::7] = lse_acc[::7] + 60.0
    lse_acc[3::11] = float("-inf")
    lse_blk[5::13] = float("-inf")
    return o_acc, lse_acc, o_blk, lse_blk


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("rows", [1, 7, 8, 1000, 4099])
def test_merge_matches_oracle(rows, d):
    o_acc, lse_acc, o_blk, lse_blk = _partials(100 + rows, rows, d)
    both_empty = (lse_acc == float("-inf")) & (lse_blk == float("-inf"))
    lse_acc[both_empty] = 0.0  # the oracle merge needs one non-empty part per row
    oa, la = o_acc.to(DEV), lse_acc.to(DEV)
    eab.attn_merge(oa, la, o_blk.to(DEV), lse_blk.to(DEV))
    torch.cuda.synchronize()
    parts = torch.stack([o_acc.double(), o_blk.double()], dim=1).view(1, rows, 2, d)
    lses = torch.stack([lse_acc.double(), lse_blk.double()], dim=1).view(1, rows, 2)
    o_ref, lse_ref = oracle.combine(parts, lses)
    o_ref, lse_ref = o_ref.view(rows, d), lse_ref.view(rows)
    assert torch.allclose(oa.double().cpu(), o_ref, rtol=2e-6, atol=2e-6)
    assert torch.allclose(la.double().cpu(), lse_ref, rtol=1e-6, atol=2e-6)


@pytest.mark.parametrize("d", [64, 128])
def test_merge_init_and_out_paths_are_exact(d):
    rows = 333
    o_acc, lse_acc, o_blk, lse_blk = _partials(7, rows, d)
    oa, la = torch.full((rows, d), 5.0, device=DEV), torch.full((rows,), 5.0, device=DEV)
    ob, lb = o_blk.to(DEV), lse_blk.to(DEV)
    eab.attn_merge(oa, la, ob, lb, init=True)  # the block itself
    out = torch.empty(rows, d, dtype=torch.bfloat16, device=DEV)
    eab.attn_merge(torch.zeros(rows, d, device=DEV), torch.zeros(rows, device=DEV), ob, lb, out=out, init=True)
    torch.cuda.synchronize()
    assert torch.equal(oa.cpu(), o_blk)
    assert torch.equal(la.cpu(), lse_blk)
    assert torch.equal(out.cpu(), o_blk.to(torch.bfloat16))
    # with `out`, o_acc is left alone and out holds the bf16 (RNE) of the merge
    oa2, la2 = o_acc.to(DEV), lse_acc.to(DEV)
    ref_o, ref_l = o_acc.to(DEV), lse_acc.to(DEV)
    eab.attn_merge(ref_o, ref_l, ob, lb)
    eab.attn_merge(oa2, la2, ob, lb, out=out)
    torch.cuda.synchronize()
    assert torch.equal(oa2.cpu(), o_acc)
    assert torch.equal(out.cpu(), ref_o.cpu().to(torch.bfloat16))
    assert torch.equal(la2.cpu(), ref_l.cpu())


def test_fwd_f32_split_last_round():
    """attn_fwd_f32 through the two launches of a non-causal call whose last
    round is split (B1 Hq32 Hkv8 N1536): bf16 of its O is attn_fwd's O bit for
    bit and the fp32 O is within tolerance of the oracle."""
    B, Hq, Hkv, N, d = 1, 32, 8, 1536, 128
    q, k, v = si.make_qkv(4150, B, Hq, Hkv, N, d)
    qg, kg, vg = q.to(DEV), k.to(DEV), v.to(DEV)
    scale = d ** -0.5
    o32 = torch.empty(B, Hq, N, d, device=DEV)
    l32 = torch.empty(B, Hq, N, device=DEV)
    eab.attn_fwd_f32(qg, kg, vg, o32, l32, False, scale)
    o16, l16 = eab.attention(qg, kg, vg, causal=False, scale=scale)
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    assert torch.equal(o32.to(torch.bfloat16), o16) and torch.equal(l32, l16)
    o_ref, lse_ref = oracle.attention(q, k, v, False, scale)
    assert_attn_close(o32, l32, o_ref, lse_ref, "fwd_f32 split B1 Hq32 Hkv8 N1536")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 130, 300, 2048])
def test_fwd_f32_is_fwd_before_rounding(N, d, causal):
    """bf16 (RNE) of attn_fwd_f32's O is attn_fwd's O bit for bit, same LSE, and the
    fp32 O itself is within tolerance of the oracle."""
    B, Hq, Hkv = 1, 4, 2
    q, k, v = si.make_qkv(41 + N, B, Hq, Hkv, N, d)
    qg, kg, vg = q.to(DEV), k.to(DEV), v.to(DEV)
    scale = d ** -0.5
    o32 = torch.empty(B, Hq, N, d, device=DEV)
    l32 = torch.empty(B, Hq, N, device=DEV)
    eab.attn_fwd_f32(qg, kg, vg, o32, l32, causal, scale)
    o16, l16 = eab.attention(qg, kg, vg, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    assert torch.equal(o32.to(torch.bfloat16), o16) and torch.equal(l32, l16)
    o_ref, lse_ref = oracle.attention(q, k, v, causal, scale)
    assert_attn_close(o32, l32, o_ref, lse_ref, f"fwd_f32 N{N} d{d} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_ring_of_one_is_attn_fwd(causal, d):
    q, k, v = si.make_qkv(31, 2, 4, 2, 300, d)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    o, lse = eab.ring_attention_emulated(q, k, v, 1, causal, d ** -0.5)
    o2, lse2 = eab.attention(q, k, v, causal=causal, scale=d ** -0.5)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


RING_CASES = [
    # B, Hq, Hkv, N, d, world, causal
    (1, 8, 2, 1024, 128, 4, False),
    (1, 8, 2, 1024, 128, 4, True),
    (2, 4, 4, 768, 64, 3, True),
    (2, 4, 1, 600, 128, 2, False),   # ragged shards of 300 rows, multi-query
    (1, 4, 2, 1200, 128, 5, True),   # shards of 240 rows
    (1, 2, 2, 512, 64, 8, True),     # 64-row shards
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,world,causal", RING_CASES)
def test_ring_matches_oracle(B, Hq, Hkv, N, d, world, causal):
    q, k, v = si.make_qkv(200 + world, B, Hq, Hkv, N, d)
    scale = d ** -0.5
    o, lse = eab.ring_attention_emulated(q.to(DEV), k.to(DEV), v.to(DEV), world, causal, scale)
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    o_ref, lse_ref = oracle.attention(q, k, v, causal, scale)
    assert_attn_close(o, lse, o_ref, lse_ref, f"ring P{world} B{B} Hq{Hq} Hkv{Hkv} N{N} d{d} causal={causal}")


def test_ring_large_logits():
    """Q x 8: the merge must track maxima that differ by far between shards."""
    B, Hq, Hkv, N, d, world = 1, 4, 4, 1024, 128, 4
    q, k, v = si.make_qkv(77, B, Hq, Hkv, N, d, 8.0)
    for causal in (False, True):
        o, lse = eab.ring_attention_emulated(q.to(DEV), k.to(DEV), v.to(DEV), world, causal, d ** -0.5)
        torch.cuda.synchronize()
        o_ref, lse_ref = oracle.attention(q, k, v, causal, d ** -0.5)
        assert_attn_close(o, lse, o_ref, lse_ref, f"ring Qx8 causal={causal}")


def test_ring_causal_rows_ignore_later_shards():
    """Changing every key/value row after shard r leaves the outputs of shards
    0..r bit for bit unchanged (later shards are skipped, never merged)."""
    B, Hq, Hkv, N, d, world = 1, 4, 2, 1024, 128, 4
    q, k, v = (t.to(DEV) for t in si.make_qkv(5, B, Hq, Hkv, N, d))
    o1, l1 = eab.ring_attention_emulated(q, k, v, world, True)
    k2, v2 = k.clone(), v.clone()
    g = torch.Generator().manual_seed(9)
    k2[:, :, 512:] = torch.randn(k2[:, :, 512:].shape, generator=g).to(torch.bfloat16).to(DEV)
    v2[:, :, 512:] = float("nan")
    o2, l2 = eab.ring_attention_emulated(q, k2, v2, world, True)
    torch.cuda.synchronize()
    assert torch.equal(o1[:, :, :512], o2[:, :, :512]) and torch.equal(l1[:, :, :512], l2[:, :, :512])

"""The library's calls captured in a CUDA graph and replayed: the replay of a
graph gives the results of the same calls made directly, bit for bit, for new
inputs copied into the captured buffers (prefill causal and not, decode with
its combine, backward, FP8 forward)."""
import pytest
import torch

import seeded_inputs as si

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import exact_attention_ring_b200 as eab  # noqa: E402

DEV = "cuda"


def _capture(fn):
    # warm the calls up on a side stream first (graph capture needs it for torch)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


@pytest.mark.parametrize("causal", [True, False])
def test_prefill_graph_replay(causal):
    B, H, N, d = 2, 8, 1000, 128
    q, k, v = (t.to(DEV) for t in si.make_qkv(7100, B, H, H, N, d))
    o, lse = torch.empty_like(q), torch.empty(B, H, N, device=DEV)
    g = _capture(lambda: eab.attn_fwd(q, k, v, o, lse, causal, d ** -0.5))
    for seed in (7101, 7102):
        q2, k2, v2 = si.make_qkv(seed, B, H, H, N, d)
        q.copy_(q2)
        k.copy_(k2)
        v.copy_(v2)
        g.replay()
        torch.cuda.synchronize()
        assert eab.attn_device_status() == 0
        o_ref, lse_ref = eab.attention(q, k, v, causal, d ** -0.5)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_decode_graph_replay():
    B, Hq, Hkv, L, d = 1, 32, 8, 20000, 128
    q, k, v = (t.to(DEV) for t in si.make_decode(7200, B, Hq, Hkv, L, d))
    S = eab.attn_decode_default_splits(B, Hq, Hkv, L)
    op, lp = torch.empty(B, Hq, S, d, device=DEV), torch.empty(B, Hq, S, device=DEV)
    o, lse = torch.empty(B, Hq, d, device=DEV, dtype=torch.bfloat16), torch.empty(B, Hq, device=DEV)

    def step():
        eab.attn_decode_splitkv(q, k, v, op, lp, S, d ** -0.5)
        eab.attn_combine(op, lp, o, lse)
    g = _capture(step)
    for seed in (7201, 7202):
        q2, k2, v2 = si.make_decode(seed, B, Hq, Hkv, L, d)
        q.copy_(q2)
        k.copy_(k2)
        v.copy_(v2)
        g.replay()
        torch.cuda.synchronize()
        assert eab.attn_device_status() == 0
        o_ref, lse_ref = eab.decode(q, k, v, d ** -0.5, num_splits=S)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_backward_and_fp8_graph_replay():
    B, H, N, d = 1, 4, 640, 128
    q, k, v = (t.to(DEV) for t in si.make_qkv(7300, B, H, H, N, d))
    do = si.make_dout(7301, B, H, N, d).to(DEV)
    o, lse = eab.attention(q, k, v, True, d ** -0.5)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    delta = torch.empty_like(lse)
    o8, lse8 = torch.empty_like(q), torch.empty_like(lse)
    q8, sq = eab.quantize_fp8(q)
    k8, sk = eab.quantize_fp8(k)
    vt8, sv = eab.quantize_fp8(v, per_plane=True, transpose=True)

    def step():
        eab.attn_bwd(q, k, v, o, lse, do, delta, dq, dk, dv, True, d ** -0.5)
        eab.attn_quant_fp8(q, q8, sq)
        eab.attn_quant_fp8(k, k8, sk)
        eab.attn_quant_fp8(v, vt8, sv, per_plane=True, transpose=True)
        eab.attn_fwd_fp8(q8, k8, vt8, sq, sk, sv, o8, lse8, True, d ** -0.5)
    g = _capture(step)
    q2, k2, v2 = si.make_qkv(7302, B, H, H, N, d)
    q.copy_(q2)
    k.copy_(k2)
    v.copy_(v2)
    o2, lse2 = eab.attention(q, k, v, True, d ** -0.5)
    o.copy_(o2)
    lse.copy_(lse2)
    g.replay()
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    dq_ref, dk_ref, dv_ref = eab.attention_backward(q, k, v, o, lse, do, True, d ** -0.5)
    o8_ref, lse8_ref = eab.attention_fp8(q, k, v, True, d ** -0.5)
    torch.cuda.synchronize()
    assert torch.equal(dq, dq_ref) and torch.equal(dk, dk_ref) and torch.equal(dv, dv_ref)
    assert torch.equal(o8, o8_ref) and torch.equal(lse8, lse8_ref)

"""GPU parity of attn_bwd (dQ, dK, dV) against the float64 oracle's backward
pass, on the same seeded bf16 inputs.

The kernels take O and LSE from attn_fwd (bf16 O, fp32 LSE) and round P and dS
to bf16 for the tensor-core products, accumulating in fp32; dQ, dK and dV are
returned in bf16. Tolerance, from that arithmetic: each gradient element is a
sum of terms each carrying a relative rounding of about 2^-9 (bf16 P or dS, and
Delta = dO . O from the bf16 O), and the result is rounded once more to bf16,
so the error relative to the tensor's RMS stays near 2^-9 ~ 2e-3. The bar is a
relative RMS error of 1e-2 and a max-abs error of 4e-2 x max|ref| per tensor,
plus an absolute floor of 1e-4 (RMS) and 1e-3 (max) for the degenerate cases
whose exact gradient is zero (a single key: dS = dP - Delta = 0), where the
kernels return fp32 rounding residue of the order of 1e-7.
"""
import pytest
import torch

import oracle
import seeded_inputs as si

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import exact_attention_ring_b200 as eab  # noqa: E402  (must load: no fallback)

DEV = "cuda"
REL_RMS = 1e-2
MAX_ABS_FRAC = 4e-2


def _close(mine, ref, what):
    mine = mine.double().cpu()
    assert torch.isfinite(mine).all(), f"{what}: non-finite gradient"
    err = mine - ref
    rms = ref.pow(2).mean().sqrt().item()
    err_rms = err.pow(2).mean().sqrt().item()
    mx = err.abs().max().item()
    peak = ref.abs().max().item()
    assert err_rms <= REL_RMS * rms + 1e-4, f"{what}: RMS error {err_rms:.3e} (RMS of ref {rms:.3e})"
    assert mx <= MAX_ABS_FRAC * peak + 1e-3, f"{what}: max-abs error {mx:.3e} (max |ref| {peak:.3e})"


def _run(B, Hq, Hkv, N, d, causal, seed, q_mult=1.0):
    q, k, v = si.make_qkv(seed, B, Hq, Hkv, N, d, q_mult)
    do = si.make_dout(seed + 1, B, Hq, N, d)
    sc = d ** -0.5
    qg, kg, vg, dog = (t.to(DEV) for t in (q, k, v, do))
    o, lse = eab.attention(qg, kg, vg, causal=causal, scale=sc)
    dq, dk, dv = eab.attention_backward(qg, kg, vg, o, lse, dog, causal=causal, scale=sc)
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    rq, rk, rv = oracle.attention_backward(q, k, v, do, causal, sc)
    tag = f"B{B} Hq{Hq} Hkv{Hkv} N{N} d{d} causal={causal}"
    _close(dq, rq, "dq " + tag)
    _close(dk, rk, "dk " + tag)
    _close(dv, rv, "dv " + tag)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,Hq,Hkv,N", [(1, 2, 2, 1), (1, 2, 2, 128), (1, 4, 2, 300), (2, 4, 1, 640),
                                        (1, 2, 2, 1000)])
def test_backward_matches_oracle(B, Hq, Hkv, N, d, causal):
    """Several 128-row tiles, a ragged tail, grouped heads (G = 1, 2, 4), N = 1."""
    _run(B, Hq, Hkv, N, d, causal, 3000 + N + d)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_large_logits(causal):
    """Q x 8 (exact in bf16): peaked rows, where P is near one-hot."""
    _run(1, 4, 4, 512, 128, causal, 3500, q_mult=8.0)


@pytest.mark.parametrize("causal", [True, False])
def test_backward_bench_shape_sampled_heads(causal):
    """The bench's backward workload (B2 H32 N2048 d128, every head in one launch
    set: 64 (batch, head) planes, several waves of the dK/dV and dQ grids),
    checked on three (batch, head) planes, each against the oracle's backward on
    that plane alone (with Hq = Hkv the gradients of a plane depend only on it)."""
    B, H, N, d = 2, 32, 2048, 128
    q, k, v = si.make_qkv(1001, B, H, H, N, d)
    do = si.make_dout(1002, B, H, N, d)
    qg, kg, vg, dog = (t.to(DEV) for t in (q, k, v, do))
    o, lse = eab.attention(qg, kg, vg, causal=causal)
    dq, dk, dv = eab.attention_backward(qg, kg, vg, o, lse, dog, causal=causal)
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    for b, h in [(0, 0), (1, 31), (0, 17)]:
        sl = (slice(b, b + 1), slice(h, h + 1))
        rq, rk, rv = oracle.attention_backward(q[sl], k[sl], v[sl], do[sl], causal, d ** -0.5)
        tag = f"bench shape causal={causal} plane ({b},{h})"
        _close(dq[sl], rq, "dq " + tag)
        _close(dk[sl], rk, "dk " + tag)
        _close(dv[sl], rv, "dv " + tag)


def test_backward_causal_first_row_has_no_dq():
    """Row 0 sees only key 0, so P_00 = 1 and dS_00 = dP_00 - Delta_0 = 0 up to
    rounding: dq of row 0 vanishes next to the other rows'."""
    q, k, v = si.make_qkv(3600, 1, 2, 2, 200, 128)
    do = si.make_dout(3601, 1, 2, 200, 128)
    qg, kg, vg, dog = (t.to(DEV) for t in (q, k, v, do))
    o, lse = eab.attention(qg, kg, vg, causal=True)
    dq, dk, dv = eab.attention_backward(qg, kg, vg, o, lse, dog, causal=True)
    torch.cuda.synchronize()
    assert dq[:, :, 0].abs().max().item() <= 1e-2 * dq.abs().max().item()


def test_backward_rejects_bad_arguments():
    q, k, v = (t.to(DEV) for t in si.make_qkv(1, 1, 2, 2, 64, 128))
    o, lse = eab.attention(q, k, v)
    delta = torch.empty_like(lse)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    with pytest.raises(eab.AttnError):
        eab.attn_bwd(q, k, v, o, lse, q, delta, dq, dk, dv, False, float("nan"))
    q96 = torch.zeros(1, 2, 64, 96, device=DEV, dtype=torch.bfloat16)
    k96 = torch.zeros(1, 2, 64, 96, device=DEV, dtype=torch.bfloat16)
    with pytest.raises(eab.AttnError):
        eab.attn_bwd(q96, k96, k96, q96, lse, q96, delta, torch.empty_like(q96), torch.empty_like(k96),
                     torch.empty_like(k96), False, 0.1)

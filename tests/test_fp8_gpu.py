"""GPU parity of the FP8 path: attn_quant_fp8 against the oracle's block
quantisation (bit for bit: codes and scales), and attn_fwd_fp8 against the
float64 oracle evaluated on the dequantised inputs.

Tolerance of the forward pass, from its arithmetic: the scores are exact E4M3
products accumulated by the tensor core in fp32 and scaled in fp32, but P is
rounded to E4M3 for the P V product. With 3 fraction bits the rounding error
of each P is within +-2^-4 of it, RMS 2^-4 / sqrt(3) = 3.6e-2, and it carries
into O with the same relative size (a float64 simulation of that rounding
alone gives 2.0e-2 to 2.5e-2 relative RMS on N(0,1) inputs). The bar: relative
RMS error <= 4e-2; max-abs error of a row <= 2^-4 max|V| (the P weights sum to
l, and each is off by at most 2^-4 of itself: |sum_j dP_j v_j| / l <= 2^-4
max|v|), plus 2^-8 max|O| for the bf16 output; LSE (which uses the fp32 P)
within 4e-3.
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
REL_RMS, LSE_ABS = 4e-2, 4e-3


def _input(seed, shape, spread):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(*shape, generator=g) * spread
    return x.to(torch.bfloat16).contiguous()


@pytest.mark.parametrize("shape", [(2, 3, 1, 64), (2, 3, 300, 128), (1, 2, 1000, 64), (1, 4, 128, 128)])
@pytest.mark.parametrize("per_plane", [False, True])
@pytest.mark.parametrize("transpose", [False, True])
def test_quant_fp8_bit_exact(shape, per_plane, transpose):
    spread = torch.tensor([0.01, 1.0, 30.0, 3.0])[: shape[1]].view(1, -1, 1, 1)
    x = _input(50 + shape[2], shape, spread)
    if shape[2] > 128:
        x[0, 1, 128:256] = 0  # an all-zero block
    codes, scales = eab.quantize_fp8(x.to(DEV), per_plane=per_plane, transpose=transpose)
    torch.cuda.synchronize()
    ref_codes, ref_scales = oracle.quant_fp8(x, per_plane=per_plane)
    assert torch.equal(scales.cpu(), ref_scales)
    c = codes.cpu()
    N = shape[2]
    if transpose:
        assert torch.equal(c[..., :N].transpose(-1, -2), ref_codes)
        assert not c[..., N:].any()
    else:
        assert torch.equal(c, ref_codes)


def _fp8_case(B, Hq, Hkv, N, causal, seed, q_mult=1.0):
    d = 128
    q, k, v = si.make_qkv(seed, B, Hq, Hkv, N, d, q_mult)
    sc = d ** -0.5
    o, lse = eab.attention_fp8(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=sc)
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    qd = oracle.dequant_fp8(*oracle.quant_fp8(q))
    kd = oracle.dequant_fp8(*oracle.quant_fp8(k))
    vd = oracle.dequant_fp8(*oracle.quant_fp8(v, per_plane=True))
    o_ref, lse_ref = oracle.attention(qd, kd, vd, causal, sc)
    err = o.double().cpu() - o_ref
    rel = (err.pow(2).mean().sqrt() / o_ref.pow(2).mean().sqrt()).item()
    mx = err.abs().max().item()
    le = (lse.double().cpu() - lse_ref).abs().max().item()
    bound = vd.abs().max().item() / 16 + o_ref.abs().max().item() / 256
    return rel, mx, le, bound


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,Hq,Hkv,N", [(1, 2, 2, 1), (1, 2, 2, 128), (1, 4, 2, 300), (2, 4, 1, 640),
                                        (1, 2, 2, 1000), (1, 160, 8, 300), (2, 50, 10, 700)])
def test_fwd_fp8_matches_oracle(B, Hq, Hkv, N, causal):
    """Small shapes run as 128-row halves without the causal mask; 160 and 100
    heads give several rounds of items, ending in a round of halves."""
    rel, mx, le, bound = _fp8_case(B, Hq, Hkv, N, causal, 4000 + N)
    tag = f"B{B} Hq{Hq} Hkv{Hkv} N{N} causal={causal}: rel {rel:.3e} max {mx:.3e} (bound {bound:.3e}) lse {le:.3e}"
    assert rel <= REL_RMS and mx <= bound and le <= LSE_ABS, tag


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_fp8_large_logits(causal):
    """Q x 8: peaked rows (the O rescale path runs when a row's maximum grows)."""
    rel, mx, le, bound = _fp8_case(1, 4, 4, 2048, causal, 4100, q_mult=8.0)
    tag = f"Qx8 causal={causal}: rel {rel:.3e} max {mx:.3e} (bound {bound:.3e}) lse {le:.3e}"
    assert rel <= REL_RMS and mx <= bound and le <= LSE_ABS, tag


@pytest.mark.parametrize("causal", [True, False])
def test_fwd_fp8_bench_shape_sampled_heads(causal):
    """The bench's FP8 workload (B2 H32 N2048 d128: 64 planes, several waves of
    query tiles), checked on three (batch, head) planes against the oracle on
    those planes' dequantised inputs (the block scales of a plane depend only on
    that plane)."""
    B, H, N, d = 2, 32, 2048, 128
    q, k, v = si.make_qkv(1001, B, H, H, N, d)
    o, lse = eab.attention_fp8(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal)
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    for b, h in [(0, 0), (1, 31), (0, 17)]:
        sl = (slice(b, b + 1), slice(h, h + 1))
        qd = oracle.dequant_fp8(*oracle.quant_fp8(q[sl].contiguous()))
        kd = oracle.dequant_fp8(*oracle.quant_fp8(k[sl].contiguous()))
        vd = oracle.dequant_fp8(*oracle.quant_fp8(v[sl].contiguous(), per_plane=True))
        o_ref, lse_ref = oracle.attention(qd, kd, vd, causal, d ** -0.5)
        err = o[sl].double().cpu() - o_ref
        rel = (err.pow(2).mean().sqrt() / o_ref.pow(2).mean().sqrt()).item()
        mx = err.abs().max().item()
        le = (lse[sl].double().cpu() - lse_ref).abs().max().item()
        bound = vd.abs().max().item() / 16 + o_ref.abs().max().item() / 256
        tag = f"plane ({b},{h}) causal={causal}: rel {rel:.3e} max {mx:.3e} (bound {bound:.3e}) lse {le:.3e}"
        assert rel <= REL_RMS and mx <= bound and le <= LSE_ABS, tag


@pytest.mark.parametrize("shape", [(2, 3, 300, 128), (1, 2, 1000, 64), (1, 1, 1, 128), (1, 4, 128, 64)])
def test_quant_fp8_rotate_bit_exact(shape):
    """Incoherent processing then block quantisation, against the oracle's
    rotation (fp32 fast Walsh-Hadamard transform) and quantisation of its
    result: codes and scales bit for bit, outlier channels included."""
    d = shape[-1]
    spread = torch.tensor([0.01, 1.0, 30.0, 3.0])[: shape[1]].view(1, -1, 1, 1)
    x = si.with_outlier_channels(_input(70 + shape[2], shape, spread))
    if shape[2] > 128:
        x[0, 1, 128:256] = 0  # an all-zero block
    sg = si.make_signs(71 + d, d)
    codes, scales = eab.quantize_fp8_rotated(x.to(DEV), sg.to(DEV))
    torch.cuda.synchronize()
    ref_codes, ref_scales = oracle.quant_fp8(oracle.hadamard_rotate(x, sg))
    assert torch.equal(scales.cpu(), ref_scales)
    assert torch.equal(codes.cpu(), ref_codes)


def _fp8_rotated_case(B, Hq, Hkv, N, causal, seed, outliers):
    d = 128
    q, k, v = si.make_qkv(seed, B, Hq, Hkv, N, d)
    if outliers:
        q, k = si.with_outlier_channels(q), si.with_outlier_channels(k)
    sg = si.make_signs(seed + 1, d)
    sc = d ** -0.5
    o, lse = eab.attention_fp8(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=sc, signs=sg.to(DEV))
    o_plain, _ = eab.attention_fp8(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=sc)
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    qd = oracle.dequant_fp8(*oracle.quant_fp8(oracle.hadamard_rotate(q, sg)))
    kd = oracle.dequant_fp8(*oracle.quant_fp8(oracle.hadamard_rotate(k, sg)))
    vd = oracle.dequant_fp8(*oracle.quant_fp8(v, per_plane=True))
    o_ref, lse_ref = oracle.attention(qd, kd, vd, causal, sc)
    o_exact, _ = oracle.attention(q, k, v, causal, sc)
    return o, lse, o_plain, o_ref, lse_ref, o_exact, vd


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("outliers", [False, True])
def test_fwd_fp8_rotated_matches_oracle(causal, outliers):
    """The FP8 forward on rotated Q and K against the oracle on the same
    dequantised rotated inputs (the FP8 bars above)."""
    o, lse, _, o_ref, lse_ref, _, vd = _fp8_rotated_case(2, 4, 2, 640, causal, 4200, outliers)
    err = o.double().cpu() - o_ref
    rel = (err.pow(2).mean().sqrt() / o_ref.pow(2).mean().sqrt()).item()
    mx = err.abs().max().item()
    le = (lse.double().cpu() - lse_ref).abs().max().item()
    bound = vd.abs().max().item() / 16 + o_ref.abs().max().item() / 256
    tag = f"rotated causal={causal} outliers={outliers}: rel {rel:.3e} max {mx:.3e} (bound {bound:.3e}) lse {le:.3e}"
    assert rel <= REL_RMS and mx <= bound and le <= LSE_ABS, tag


def test_incoherent_processing_lowers_gpu_fp8_error():
    """What the rotation is for (FlashAttention-3 page: lower FP8 error with
    incoherent processing): with outlier channels in Q and K, the GPU's FP8
    forward with rotation is at least twice as close to exact attention on the
    bf16 inputs as without."""
    o, _, o_plain, _, _, o_exact, _ = _fp8_rotated_case(1, 4, 4, 512, False, 4300, True)
    rms = o_exact.pow(2).mean().sqrt().item()
    rot = (o.double().cpu() - o_exact).pow(2).mean().sqrt().item() / rms
    plain = (o_plain.double().cpu() - o_exact).pow(2).mean().sqrt().item() / rms
    assert rot * 2 <= plain, (plain, rot)


def test_fwd_fp8_rejects_unsupported_head_dim():
    q = torch.zeros(1, 2, 64, 64, device=DEV, dtype=torch.uint8)
    s = torch.ones(1, 2, 1, device=DEV)
    o = torch.empty(1, 2, 64, 64, device=DEV, dtype=torch.bfloat16)
    lse = torch.empty(1, 2, 64, device=DEV)
    vt = torch.zeros(1, 2, 64, 128, device=DEV, dtype=torch.uint8)
    with pytest.raises(eab.AttnError):
        eab.attn_fwd_fp8(q, q, vt, s, s, s, o, lse, False, 0.125)

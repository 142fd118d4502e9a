"""Pins for the float64 oracle: facts fixed by the pages and by mathematics.

None of these re-types the oracle's own formula. Each pin compares the oracle
with something independent of it: a closed form, an invariant of the
definition, an independent library routine (torch's float64 CPU
scaled_dot_product_attention, scipy's softmax / logsumexp), or another
oracle function that follows a different algorithm (the blockwise online
recurrence of the "递归计算softmax" section of "1-Flash-Attention.md").

The mutation test at the bottom builds oracle variants with one planted
mistake each (a dropped scale, a wrong GQA grouping, a causal off-by-one, a
log2 LSE, a missing rescale, a plain-average merge, a transposed K, a dropped
key, unnormalised partials, E4M3 rounding toward zero, a rotation missing its
1/sqrt(d)) and checks that at least one pin fails on each.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle

TOL = 1e-12


def _rand(seed, *shape):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64)


def _sdpa(q, k, v, causal, scale):
    return F.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=scale, enable_gqa=True)


def _lse_lib(q, k, causal, scale):
    """LSE by scipy's logsumexp over masked scores (library routine)."""
    B, Hq, N, d = q.shape
    G = Hq // k.shape[1]
    kk = k.repeat_interleave(G, dim=1)
    s = (q @ kk.transpose(-1, -2)).numpy() * scale
    if causal:
        mask = np.triu(np.ones((N, k.shape[2]), dtype=bool), 1)
        s = np.where(mask, -np.inf, s)
    return torch.from_numpy(scipy.special.logsumexp(s, axis=-1))


# ---------------------------------------------------------------- pins ----

def pin_probs_are_distributions(plant=0):
    """Softmax rows are probability vectors; causal rows put no mass past i."""
    q, k, v = _rand(1, 1, 2, 9, 4), _rand(2, 1, 2, 9, 4), _rand(3, 1, 2, 9, 4)
    for causal in (False, True):
        _, _, p = oracle.attention(q, k, v, causal, 0.7, want_probs=True, plant=plant)
        assert torch.all(p >= 0)
        assert torch.allclose(p.sum(-1), torch.ones(1, 2, 9, dtype=torch.float64), atol=1e-14, rtol=0)
        if causal:
            assert torch.all(torch.triu(p[0, 0], 1) == 0)


def pin_constant_v(plant=0):
    """v_j = c for every j gives O_i = c for every row (weights sum to one)."""
    q, k = _rand(4, 2, 3, 17, 8), _rand(5, 2, 3, 17, 8)
    c = _rand(6, 8)
    v = c.expand(2, 3, 17, 8).contiguous()
    for causal in (False, True):
        o, _ = oracle.attention(q, k, v, causal, 0.35, plant=plant)
        assert torch.allclose(o, c.expand_as(o), atol=1e-14, rtol=0)


def pin_causal_first_row(plant=0):
    """Causal row 0 sees only key 0: O[0] = V[0], LSE[0] = scale * q0.k0."""
    q, k, v = _rand(7, 1, 2, 12, 5), _rand(8, 1, 2, 12, 5), _rand(9, 1, 2, 12, 5)
    o, lse = oracle.attention(q, k, v, True, 0.5, plant=plant)
    assert torch.allclose(o[:, :, 0], v[:, :, 0], atol=1e-15, rtol=0)
    dots = torch.tensor([[math.fsum((q[0, h, 0] * k[0, h, 0]).tolist()) for h in range(2)]], dtype=torch.float64)
    assert torch.allclose(lse[:, :, 0], 0.5 * dots, atol=1e-14, rtol=0)


def pin_single_key(plant=0):
    """N = 1: the only key gets weight one, so O = V and LSE = scale * q.k."""
    q, k, v = _rand(10, 3, 4, 1, 6), _rand(11, 3, 2, 1, 6), _rand(12, 3, 2, 1, 6)
    for causal in (False, True):
        o, lse = oracle.attention(q, k, v, causal, 1.3, plant=plant)
        vv = v.repeat_interleave(2, dim=1)
        kk = k.repeat_interleave(2, dim=1)
        assert torch.allclose(o, vv, atol=1e-15, rtol=0)
        assert torch.allclose(lse, 1.3 * (q * kk).sum(-1), atol=1e-13, rtol=0)


def pin_two_keys_closed_form(plant=0):
    """Scores {0, t*ln2}: weights 1/(1+2^t) and 2^t/(1+2^t), LSE = ln(1+2^t)."""
    scale = 0.25
    for t in (-3, 0, 1, 5):
        q = torch.ones(1, 1, 2, 1, dtype=torch.float64)
        k = torch.tensor([0.0, t * math.log(2) / scale], dtype=torch.float64).view(1, 1, 2, 1)
        v = torch.tensor([2.0, -6.0], dtype=torch.float64).view(1, 1, 2, 1)
        o, lse = oracle.attention(q, k, v, False, scale, plant=plant)
        w1 = 2.0 ** t / (1 + 2.0 ** t)
        want = (1 - w1) * 2.0 + w1 * -6.0
        assert abs(o[0, 0, 0, 0].item() - want) < 1e-14
        assert abs(lse[0, 0, 0].item() - math.log1p(2.0 ** t)) < 1e-14
        # causal: row 0 sees key 0 only, row 1 sees both
        o, lse = oracle.attention(q, k, v, True, scale, plant=plant)
        assert abs(o[0, 0, 0, 0].item() - 2.0) < 1e-15
        assert abs(o[0, 0, 1, 0].item() - want) < 1e-14


def pin_identical_keys(plant=0):
    """All keys equal: uniform weights, O = mean(V), LSE = s + ln(N)."""
    N, d = 11, 3
    q = _rand(13, 1, 1, N, d)
    k = _rand(14, d).expand(1, 1, N, d).contiguous()
    v = _rand(15, 1, 1, N, d)
    o, lse = oracle.attention(q, k, v, False, 0.9, plant=plant)
    assert torch.allclose(o[0, 0], v[0, 0].mean(0).expand(N, d), atol=1e-14, rtol=0)
    s = 0.9 * (q[0, 0] @ k[0, 0, 0])
    assert torch.allclose(lse[0, 0], s + math.log(N), atol=1e-13, rtol=0)


def pin_library_sdpa(plant=0):
    """Matches torch's float64 CPU SDPA (O) and scipy logsumexp (LSE), with GQA."""
    cases = [(1, 1, 1, 7, 3), (2, 4, 2, 13, 5), (1, 6, 3, 9, 4), (1, 4, 1, 16, 8), (2, 2, 2, 5, 2)]
    for i, (B, Hq, Hkv, N, d) in enumerate(cases):
        q, k, v = _rand(20 + i, B, Hq, N, d), _rand(30 + i, B, Hkv, N, d), _rand(40 + i, B, Hkv, N, d)
        for causal in (False, True):
            scale = 0.3 + 0.2 * i
            o, lse = oracle.attention(q, k, v, causal, scale, plant=plant)
            assert torch.allclose(o, _sdpa(q, k, v, causal, scale), atol=1e-12, rtol=0)
            assert torch.allclose(lse, _lse_lib(q, k, causal, scale), atol=1e-12, rtol=0)


def pin_brute_force_tiny(plant=0):
    """Exhaustive tiny shapes against scipy's softmax, row by row."""
    seed = 100
    for N in range(1, 6):
        for d in (1, 2, 3):
            for Hq, Hkv in ((1, 1), (2, 1), (2, 2), (4, 2)):
                seed += 1
                q, k, v = _rand(seed, 1, Hq, N, d), _rand(seed + 1000, 1, Hkv, N, d), _rand(seed + 2000, 1, Hkv, N, d)
                for causal in (False, True):
                    o, _ = oracle.attention(q, k, v, causal, 0.8, plant=plant)
                    G = Hq // Hkv
                    for h in range(Hq):
                        for i in range(N):
                            J = i + 1 if causal else N
                            s = 0.8 * (k[0, h // G, :J] @ q[0, h, i]).numpy()
                            want = scipy.special.softmax(s) @ v[0, h // G, :J].numpy()
                            assert np.allclose(o[0, h, i].numpy(), want, atol=1e-13, rtol=0)


def pin_blockwise_equals_direct(plant=0):
    """The online recurrence over key blocks reaches the direct result for any block size."""
    q, k, v = _rand(50, 2, 4, 70, 8), _rand(51, 2, 2, 70, 8), _rand(52, 2, 2, 70, 8)
    q = q * 6  # large logits: the running max moves a lot between blocks
    for causal in (False, True):
        o, lse = oracle.attention(q, k, v, causal, 0.5, plant=plant)
        for bk in (1, 3, 7, 64, 70):
            ob, lb = oracle.attention_blockwise(q, k, v, causal, 0.5, bk, plant=plant)
            assert torch.allclose(ob, o, atol=1e-12, rtol=1e-12)
            assert torch.allclose(lb, lse, atol=1e-12, rtol=1e-12)


def pin_invariants(plant=0):
    """Joint key/value permutation, key shift and GQA replication invariants."""
    B, Hq, Hkv, N, d = 1, 4, 2, 10, 6
    q, k, v = _rand(60, B, Hq, N, d), _rand(61, B, Hkv, N, d), _rand(62, B, Hkv, N, d)
    o, lse = oracle.attention(q, k, v, False, 0.6, plant=plant)
    perm = torch.randperm(N, generator=torch.Generator().manual_seed(63))
    op, lp = oracle.attention(q, k[:, :, perm].contiguous(), v[:, :, perm].contiguous(), False, 0.6, plant=plant)
    assert torch.allclose(op, o, atol=1e-13, rtol=0) and torch.allclose(lp, lse, atol=1e-13, rtol=0)
    u = _rand(64, d)
    os_, ls_ = oracle.attention(q, (k + u).contiguous(), v, False, 0.6, plant=plant)
    assert torch.allclose(os_, o, atol=1e-12, rtol=0)
    assert torch.allclose(ls_, lse + 0.6 * (q @ u), atol=1e-12, rtol=0)
    G = Hq // Hkv
    for causal in (False, True):
        og, lg = oracle.attention(q, k, v, causal, 0.6, plant=plant)
        om, lm = oracle.attention(q, k.repeat_interleave(G, 1).contiguous(),
                                  v.repeat_interleave(G, 1).contiguous(), causal, 0.6, plant=plant)
        assert torch.equal(og, om) and torch.equal(lg, lm)
        # shifting V of key/value head 1 by +1 moves exactly query heads G..2G-1 by +1
        v2 = v.clone()
        v2[:, 1] += 1.0
        og2, _ = oracle.attention(q, k, v2, causal, 0.6, plant=plant)
        assert torch.equal(og2[:, :G], og[:, :G])
        assert torch.allclose(og2[:, G:], og[:, G:] + 1.0, atol=1e-13, rtol=0)


def pin_decode_and_combine(plant=0):
    """Decode = last row of causal prefill; merging any split of the keys = direct."""
    B, Hq, Hkv, L, d = 2, 4, 2, 37, 5
    q, k, v = _rand(70, B, Hq, L, d), _rand(71, B, Hkv, L, d), _rand(72, B, Hkv, L, d)
    o_pre, l_pre = oracle.attention(q, k, v, True, 0.45, plant=plant)
    qd = q[:, :, L - 1].contiguous()
    od, ld = oracle.decode(qd, k, v, 0.45)
    assert torch.allclose(od, o_pre[:, :, L - 1], atol=1e-13, rtol=0)
    assert torch.allclose(ld, l_pre[:, :, L - 1], atol=1e-13, rtol=0)
    for S, chunk in ((1, 37), (2, 19), (5, 8), (8, 5), (40, 1), (7, 8)):  # (7, 8): empty splits
        op, lp = oracle.decode_partials(qd, k, v, 0.45, S, chunk, plant=plant)
        oc, lc = oracle.combine(op, lp, plant=plant)
        assert torch.allclose(oc, od, atol=1e-13, rtol=0)
        assert torch.allclose(lc, ld, atol=1e-13, rtol=0)


def pin_bf16_inputs_widen_exactly(plant=0):
    """bf16 inputs give the same answer as the same values passed as float64."""
    q, k, v = (_rand(s, 1, 2, 9, 8).to(torch.bfloat16) for s in (80, 81, 82))
    ob, lb = oracle.attention(q, k, v, True, 0.3, plant=plant)
    od, ld = oracle.attention(q.double(), k.double(), v.double(), True, 0.3, plant=plant)
    assert torch.equal(ob, od) and torch.equal(lb, ld)


def pin_fp16_inputs_widen_exactly(plant=0):
    """fp16 inputs: the oracle's own binary16 decoding agrees with torch's on all
    65,536 bit patterns, and fp16 inputs give the same answer as their values
    passed as float64."""
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.float16)
    w, ref = oracle.widen(bits), bits.to(torch.float64)
    nan = torch.isnan(ref)
    assert torch.equal(torch.isnan(w), nan) and torch.equal(w[~nan], ref[~nan])
    q, k, v = (_rand(s, 1, 2, 9, 8).to(torch.float16) for s in (83, 84, 85))
    oh, lh = oracle.attention(q, k, v, True, 0.3, plant=plant)
    od, ld = oracle.attention(q.double(), k.double(), v.double(), True, 0.3, plant=plant)
    assert torch.equal(oh, od) and torch.equal(lh, ld)


def test_bf16_widening_matches_torch():
    """The oracle's bf16 decoding agrees with torch's on all 65,536 bit patterns."""
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    w, ref = oracle.widen(bits), bits.to(torch.float64)
    nan = torch.isnan(ref)
    assert torch.equal(torch.isnan(w), nan) and torch.equal(w[~nan], ref[~nan])


def pin_row_sampling(plant=0):
    """Computing a subset of rows gives exactly those rows of the full result."""
    q, k, v = _rand(90, 2, 3, 20, 4), _rand(91, 2, 3, 20, 4), _rand(92, 2, 3, 20, 4)
    o, lse = oracle.attention(q, k, v, True, 0.5, plant=plant)
    rows = torch.tensor([0, 19, 20, 57, 119])
    orr, lr = oracle.attention(q, k, v, True, 0.5, rows=rows, plant=plant)
    assert torch.equal(orr, o.reshape(-1, 4)[rows]) and torch.equal(lr, lse.reshape(-1)[rows])


def pin_e4m3_codec_matches_torch(plant=0):
    """E4M3 values of all 256 codes, and the nearest-even rounding of floats
    (random values across the range, and every exact midpoint between two
    neighbouring values), against torch's float8_e4m3fn conversion."""
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64)
    mine = oracle.e4m3_decode(codes)
    nan = torch.isnan(ref)
    assert torch.isnan(mine[nan]).all() and torch.equal(mine[~nan], ref[~nan])
    g = torch.Generator().manual_seed(60)
    x = torch.cat([torch.randn(20000, generator=g) * 60, torch.randn(20000, generator=g) * 0.02,
                   (torch.rand(20000, generator=g) * 2 - 1) * 448]).clamp(-448, 448)
    pos = torch.unique(ref[~nan].abs()).sort().values
    mid = ((pos[1:] + pos[:-1]) / 2).to(torch.float32)
    x = torch.cat([x, mid, -mid])
    assert torch.equal(oracle.e4m3_encode(x, plant=plant), x.to(torch.float8_e4m3fn).view(torch.uint8))
    # saturation past the largest finite value
    big = torch.tensor([448.0, 470.0, 1e6, -1e6])
    assert oracle.e4m3_decode(oracle.e4m3_encode(big, plant=plant)).tolist() == [448.0, 448.0, 448.0, -448.0]


def pin_quant_fp8_blocks(plant=0):
    """Block quantisation: scale = amax / 448 in fp32 per 128-row block (or per
    plane), codes = torch's E4M3 rounding of x / scale in fp32; the largest
    element of a block lands on +-448 exactly; an all-zero block has scale 1."""
    g = torch.Generator().manual_seed(61)
    x = (torch.randn(2, 3, 300, 64, generator=g) * torch.tensor([0.01, 1.0, 30.0]).view(1, 3, 1, 1)).to(torch.bfloat16)
    x[1, 2, 128:256] = 0
    for per_plane in (False, True):
        codes, scales = oracle.quant_fp8(x, per_plane=per_plane, plant=plant)
        xf = x.float()
        blocks = [xf[..., i:i + 128, :].abs().amax(dim=(-1, -2)) for i in range(0, 300, 128)]
        amax = torch.stack(blocks, dim=-1)
        if per_plane:
            amax = amax.amax(dim=-1, keepdim=True).expand_as(amax)
        want = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        assert torch.equal(scales, want)
        rep = scales.repeat_interleave(128, dim=-1)[..., :300].unsqueeze(-1)
        assert torch.equal(codes, (xf / rep).to(torch.float8_e4m3fn).view(torch.uint8))
        deq = oracle.dequant_fp8(codes, scales)
        if not per_plane:
            top = deq.abs().amax(dim=-1)
            for i, s0 in enumerate(range(0, 300, 128)):
                blk = top[..., s0:s0 + 128].amax(dim=-1)
                nz = amax[..., i] > 0
                assert torch.equal(blk[nz], (448.0 * scales[..., i].double())[nz])
    assert torch.equal(oracle.quant_fp8(x)[1][1, 2, 1], torch.tensor(1.0))


def pin_hadamard_rotation(plant=0):
    """The incoherent-processing rotation against scipy's Hadamard matrix (within
    fp32 rounding), its orthogonality (norms and dot products kept, so Q K^T is
    unchanged), and the exact spreading of a one-hot outlier at d = 64."""
    import scipy.linalg
    g = torch.Generator().manual_seed(62)
    for d in (64, 128):
        x = torch.randn(40, d, generator=g)
        z = torch.randn(40, d, generator=g)
        sg = torch.where(torch.rand(d, generator=g) < 0.5, -1.0, 1.0)
        y = oracle.hadamard_rotate(x, sg, plant=plant).double()
        w = oracle.hadamard_rotate(z, sg, plant=plant).double()
        H = torch.from_numpy(scipy.linalg.hadamard(d)).double()
        ref = (x.double() * sg.double()) @ H.T / math.sqrt(d)
        assert (y - ref).abs().max().item() <= 1e-6 * ref.abs().max().item() * math.sqrt(d)
        assert torch.allclose(y.norm(dim=-1), x.double().norm(dim=-1), rtol=1e-6, atol=0)
        assert torch.allclose((y * w).sum(-1), (x.double() * z.double()).sum(-1), rtol=0, atol=1e-4)
    one_hot = torch.zeros(1, 64)
    one_hot[0, 5] = 100.0
    y = oracle.hadamard_rotate(one_hot, torch.ones(64), plant=plant)
    assert torch.equal(y.abs(), torch.full((1, 64), 12.5))


PINS = [pin_probs_are_distributions, pin_constant_v, pin_causal_first_row, pin_single_key,
        pin_two_keys_closed_form, pin_identical_keys, pin_library_sdpa, pin_brute_force_tiny,
        pin_blockwise_equals_direct, pin_invariants, pin_decode_and_combine,
        pin_bf16_inputs_widen_exactly, pin_fp16_inputs_widen_exactly, pin_row_sampling,
        pin_e4m3_codec_matches_torch, pin_quant_fp8_blocks, pin_hadamard_rotation]


def test_backward_matches_autograd():
    """The backward pass against torch's float64 autograd of its SDPA (causal
    and not, grouped heads)."""
    g = torch.Generator().manual_seed(120)
    B, Hq, Hkv, N, d = 2, 4, 2, 9, 6
    for causal in (False, True):
        q = torch.randn(B, Hq, N, d, generator=g, dtype=torch.float64, requires_grad=True)
        k = torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64, requires_grad=True)
        v = torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64, requires_grad=True)
        do = torch.randn(B, Hq, N, d, generator=g, dtype=torch.float64)
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=0.35, enable_gqa=True)
        o.backward(do)
        dq, dk, dv = oracle.attention_backward(q.detach(), k.detach(), v.detach(), do, causal, 0.35)
        for mine, ref in ((dq, q.grad), (dk, k.grad), (dv, v.grad)):
            assert torch.allclose(mine, ref, atol=1e-12, rtol=0)


def test_backward_matches_finite_differences():
    """Central differences of sum(dO * O) through the oracle's own forward pass."""
    g = torch.Generator().manual_seed(121)
    B, Hq, Hkv, N, d, sc = 1, 2, 1, 5, 3, 0.6
    q, k, v, do = (torch.randn(*sh, generator=g, dtype=torch.float64)
                   for sh in ((B, Hq, N, d), (B, Hkv, N, d), (B, Hkv, N, d), (B, Hq, N, d)))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, True, sc)
    eps = 1e-6

    def loss(qq, kk, vv):
        return float((oracle.attention(qq, kk, vv, True, sc)[0] * do).sum())

    for t, grad, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        for idx in range(t.numel()):
            plus, minus = [q.clone(), k.clone(), v.clone()], [q.clone(), k.clone(), v.clone()]
            plus[which].view(-1)[idx] += eps
            minus[which].view(-1)[idx] -= eps
            fd = (loss(*plus) - loss(*minus)) / (2 * eps)
            assert abs(fd - grad.view(-1)[idx].item()) < 1e-6


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


PLANTS = {1: "scale dropped", 2: "GQA head h % Hkv", 3: "causal off by one", 4: "LSE in log2",
          5: "recurrence without rescale", 6: "merge by plain average", 7: "K read transposed",
          8: "one key dropped", 9: "partials not normalised", 10: "E4M3 rounding toward zero",
          11: "rotation without 1/sqrt(d)"}


@pytest.mark.parametrize("plant", sorted(PLANTS), ids=[PLANTS[p] for p in sorted(PLANTS)])
def test_planted_mistake_is_caught(plant):
    caught = []
    for pin in PINS:
        try:
            pin(plant=plant)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches planted mistake {plant} ({PLANTS[plant]})"


def test_incoherent_processing_lowers_fp8_error():
    """What the rotation is for (FlashAttention-3 page: FP8 error lowered by
    incoherent processing): with two outlier channels in Q and K, attention on
    block-quantised E4M3 inputs is at least twice as close to the exact result
    when Q and K are rotated first."""
    import seeded_inputs as si
    q, k, v = si.make_qkv(11, 1, 2, 2, 256, 128)
    qf, kf = q.float(), k.float()
    qf[..., 3] *= 20
    kf[..., 3] *= 20
    qf[..., 77] *= 15
    kf[..., 77] *= 15
    qf, kf = qf.to(torch.bfloat16), kf.to(torch.bfloat16)
    sc = 128 ** -0.5
    o_ref, _ = oracle.attention(qf, kf, v, False, sc)
    vd = oracle.dequant_fp8(*oracle.quant_fp8(v, per_plane=True))
    g = torch.Generator().manual_seed(5)
    sg = torch.where(torch.rand(128, generator=g) < 0.5, -1.0, 1.0)

    def rel_err(qq, kk):
        qd = oracle.dequant_fp8(*oracle.quant_fp8(qq))
        kd = oracle.dequant_fp8(*oracle.quant_fp8(kk))
        o, _ = oracle.attention(qd, kd, vd, False, sc)
        return ((o - o_ref).pow(2).mean().sqrt() / o_ref.pow(2).mean().sqrt()).item()

    plain = rel_err(qf, kf)
    rotated = rel_err(oracle.hadamard_rotate(qf, sg), oracle.hadamard_rotate(kf, sg))
    assert rotated * 2 <= plain, (plain, rotated)

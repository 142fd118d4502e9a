"""GPU parity of attn_fwd against the float64 oracle (same seeded inputs).

Small shapes are compared element by element in full (several tiles plus
ragged tails); the full-size workloads are compared on sampled rows (row 0,
the last row, rows on both sides of every 128-row tile boundary and random
rows) in the same launch configuration the bench times. Masking and the
grouped-query head mapping are checked bit for bit.
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


def run_gpu(q, k, v, causal, scale):
    o, lse = eab.attention(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    return o, lse


def check_full(B, Hq, Hkv, N, d, causal, seed, q_mult=1.0, scale=None):
    q, k, v = si.make_qkv(seed, B, Hq, Hkv, N, d, q_mult)
    scale = scale or d ** -0.5
    o, lse = run_gpu(q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attention(q, k, v, causal, scale)
    return assert_attn_close(o, lse, o_ref, lse_ref, f"B{B} Hq{Hq} Hkv{Hkv} N{N} d{d} causal={causal}")


def check_sampled(shape: si.PrefillShape, per_slice=128, max_slices=4):
    q, k, v = si.make_qkv(shape.seed, shape.B, shape.Hq, shape.Hkv, shape.N, shape.d, shape.q_mult)
    o, lse = run_gpu(q, k, v, shape.causal, shape.scale)
    rows = si.sample_rows(shape.seed + 7, shape.B, shape.Hq, shape.N, per_slice=per_slice, max_slices=max_slices)
    o_ref, lse_ref = oracle.attention(q, k, v, shape.causal, shape.scale, rows=rows)
    o_s = o.reshape(-1, shape.d)[rows.to(DEV)]
    l_s = lse.reshape(-1)[rows.to(DEV)]
    return assert_attn_close(o_s, l_s, o_ref, lse_ref, shape.name)


# ------------------------------------------------------------ full checks --

def test_single_head_config():
    s = si.SINGLE_HEAD
    check_full(s.B, s.Hq, s.Hkv, s.N, s.d, s.causal, s.seed)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 63, 127, 128, 129, 255, 300, 640, 1000])
def test_ragged_lengths(N, causal, d):
    check_full(1, 2, 2, N, d, causal, seed=2000 + N)


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (4, 1), (6, 3), (8, 8)])
@pytest.mark.parametrize("causal", [False, True])
def test_grouped_heads(Hq, Hkv, causal):
    check_full(2, Hq, Hkv, 200, 128, causal, seed=3000 + Hq * 10 + Hkv)


@pytest.mark.parametrize("causal", [False, True])
def test_large_logits_small(causal):
    check_full(1, 2, 2, 600, 128, causal, seed=3100, q_mult=8.0)
    check_full(1, 2, 2, 600, 64, causal, seed=3101, q_mult=16.0)


def test_nondefault_scale():
    check_full(1, 2, 1, 300, 64, True, seed=3200, scale=0.37)


# ------------------------------------------------- full-size, sampled rows --

@pytest.mark.parametrize("shape", si.LLAMA7B, ids=[s.name for s in si.LLAMA7B])
def test_llama7b_shape(shape):
    check_sampled(shape)


SWEEP = si.sweep_shapes()


@pytest.mark.parametrize("shape", SWEEP, ids=[s.name for s in SWEEP])
def test_sweep(shape):
    check_sampled(shape, per_slice=64, max_slices=2)


@pytest.mark.parametrize("shape", si.GQA, ids=[s.name for s in si.GQA])
def test_gqa_mqa(shape):
    check_sampled(shape, per_slice=96, max_slices=4)


# ------------------------------------------------------------ bit-exact ----

@pytest.mark.parametrize("d", [64, 128])
def test_causal_first_row_is_v0(d):
    """Row 0 sees only key 0: p = exp2(0) = 1, l = 1, so O[0] = V[0] exactly."""
    q, k, v = si.make_qkv(4000, 2, 4, 2, 300, d)
    o, lse = run_gpu(q, k, v, True, d ** -0.5)
    want = v.repeat_interleave(2, dim=1)[:, :, 0].to(DEV)
    assert torch.equal(o[:, :, 0], want)
    dots = (q[:, :, 0].double() * k.repeat_interleave(2, dim=1)[:, :, 0].double()).sum(-1) * d ** -0.5
    assert torch.allclose(lse[:, :, 0].double().cpu(), dots, atol=1e-4, rtol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_single_key_gives_v(causal):
    q, k, v = si.make_qkv(4100, 3, 4, 4, 1, 128)
    o, _ = run_gpu(q, k, v, causal, 0.088)
    assert torch.equal(o.cpu(), v)


@pytest.mark.parametrize("d", [64, 128])
def test_future_keys_do_not_leak(d):
    """Causal: changing keys/values after row i leaves rows <= i bit-identical,
    and keys in tiles past the diagonal are never read (NaN poison stays out)."""
    N = 512
    q, k, v = si.make_qkv(4200, 1, 2, 2, N, d)
    o, lse = run_gpu(q, k, v, True, d ** -0.5)
    i = 200  # inside the second tile: keys 201..255 share the diagonal tile
    k2, v2 = k.clone(), v.clone()
    k2[:, :, i + 1:] = k2[:, :, i + 1:] * -3 + 1
    v2[:, :, i + 1:] = v2[:, :, i + 1:] * 5 - 2
    o2, lse2 = run_gpu(q, k2, v2, True, d ** -0.5)
    assert torch.equal(o2[:, :, : i + 1], o[:, :, : i + 1])
    assert torch.equal(lse2[:, :, : i + 1], lse[:, :, : i + 1])
    k3, v3 = k.clone(), v.clone()
    k3[:, :, 256:] = float("nan")
    v3[:, :, 256:] = float("nan")
    o3, lse3 = run_gpu(q, k3, v3, True, d ** -0.5)
    assert torch.equal(o3[:, :, :256], o[:, :, :256])
    assert torch.equal(lse3[:, :, :256], lse[:, :, :256])


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_equals_replicated_mha(causal):
    """Query head h reads key/value head h // G: the grouped run equals an MHA
    run on repeat_interleave'd K/V bit for bit."""
    q, k, v = si.make_qkv(4300, 2, 8, 2, 333, 128)
    og, lg = run_gpu(q, k, v, causal, 0.09)
    om, lm = run_gpu(q, k.repeat_interleave(4, 1).contiguous(), v.repeat_interleave(4, 1).contiguous(), causal, 0.09)
    assert torch.equal(og, om) and torch.equal(lg, lm)


def test_outputs_only_in_bounds():
    """Writes stay inside o and lse: canaries around both buffers survive."""
    B, H, N, d = 1, 2, 200, 128
    q, k, v = si.make_qkv(4400, B, H, H, N, d)
    pad = 4096
    o_buf = torch.full((pad * 2 + B * H * N * d,), 7.0, dtype=torch.bfloat16, device=DEV)
    l_buf = torch.full((pad * 2 + B * H * N,), 7.0, dtype=torch.float32, device=DEV)
    o = o_buf[pad:pad + B * H * N * d].view(B, H, N, d)
    lse = l_buf[pad:pad + B * H * N].view(B, H, N)
    eab.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), o, lse, True, d ** -0.5)
    torch.cuda.synchronize()
    assert torch.all(o_buf[:pad] == 7.0) and torch.all(o_buf[-pad:] == 7.0)
    assert torch.all(l_buf[:pad] == 7.0) and torch.all(l_buf[-pad:] == 7.0)


def test_repeatable():
    q, k, v = si.make_qkv(4500, 2, 4, 4, 700, 128)
    o1, l1 = run_gpu(q, k, v, True, 0.088)
    o2, l2 = run_gpu(q, k, v, True, 0.088)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_repeatable_large_logits_many_tiles():
    """Non-causal, Q x 8, 16 key tiles per row: mid-stream rescales skew the
    softmax warps' timing; repeated runs must agree bit for bit."""
    q, k, v = si.make_qkv(4600, 2, 32, 32, 2048, 128, 8.0)
    o1, l1 = run_gpu(q, k, v, False, 128 ** -0.5)
    for _ in range(3):
        o2, l2 = run_gpu(q, k, v, False, 128 ** -0.5)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("d", [64, 128])
def test_split_last_round(d):
    """A non-causal problem whose last round holds at most half as many query
    blocks as there are SMs runs that round as a second launch of 128-row items,
    each tile of a CTA over half of the keys, merged in the epilogue. B1 H32
    N1536: 192 blocks, so on 148 SMs the first launch takes 148 and the split
    launch the other 44 (88 items). Every row against the oracle."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    blocks = 32 * 1536 // 256
    assert 2 * (blocks % sms) <= sms, "shape chosen for a split last round on this GPU"
    check_full(1, 32, 32, 1536, d, False, 6300 + d)


def test_split_last_round_ragged_odd_key_tiles():
    """Split items with an odd number of key tiles (tile 1 takes the extra one,
    with no turn) and a ragged last key tile in tile 1's half: N = 1100 gives
    nine key tiles, 4 for tile 0 and 5 for tile 1; B1 H8 gives 40 blocks, all
    split."""
    check_full(1, 8, 8, 1100, 128, False, 6350)
    check_full(1, 8, 2, 1100, 64, False, 6351)


@pytest.mark.parametrize("shape", [(2, 32, 2048), (1, 8, 1100)], ids=["two_launches", "split_only"])
def test_split_launch_stream_order(shape):
    """The split launch of a non-causal call starts its blocks in the tail of
    the call's first launch and waits for it only before it exits; a split
    launch with no first launch waits for the previous kernel at its start.
    Inputs written by the kernel just before the call, and a copy of the
    outputs made by the kernel just after it, must see the stream's order."""
    B, H, N = shape
    d = 128
    q, k, v = (t.to(DEV) for t in si.make_qkv(6400 + N, B, H, H, N, d))
    o_ref, lse_ref = eab.attention(q, k, v, causal=False)
    torch.cuda.synchronize()
    q_in = torch.full_like(q, float("nan"))
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device=DEV)
    for _ in range(3):
        q_in.fill_(float("nan"))
        o.fill_(float("nan"))
        q_in.copy_(q)  # written by the kernel right before the call
        eab.attn_fwd(q_in, k, v, o, lse, False, d ** -0.5)
        o_after, lse_after = o.clone(), lse.clone()  # read by the kernel right after it
        torch.cuda.synchronize()
        assert eab.attn_device_status() == 0
        assert torch.equal(o_after, o_ref) and torch.equal(lse_after, lse_ref)


def test_work_counter_slots_are_reused_and_reset():
    """Non-causal launches hand out work items from a per-launch counter slot
    that the launch's last CTA resets. 70 launches in a row (more than the 64
    slots, so slots are used twice) on a problem with more items than CTAs, each
    into a NaN-poisoned output, all give the first launch's result bit for bit:
    every item is computed once by one CTA whichever CTA takes it."""
    B, H, N, d = 2, 32, 1024, 128  # 4 query blocks x 64 planes = 256 items > 148 CTAs
    q, k, v = (t.to(DEV) for t in si.make_qkv(6100, B, H, H, N, d))
    refs = {c: eab.attention(q, k, v, causal=c) for c in (False, True)}
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, device=DEV)
    for i in range(70):
        causal = i % 5 == 4  # mostly non-causal launches, which take items from the counter
        o.fill_(float("nan"))
        lse.fill_(float("nan"))
        eab.attn_fwd(q, k, v, o, lse, causal, d ** -0.5)
        torch.cuda.synchronize()
        assert torch.equal(o, refs[causal][0]) and torch.equal(lse, refs[causal][1]), f"launch {i}"
    assert eab.attn_device_status() == 0


def test_concurrent_launches_on_two_streams():
    """Launches in flight at the same time on two streams take different counter
    slots and do not steal each other's work items."""
    B, H, N, d = 2, 32, 1536, 128
    q, k, v = (t.to(DEV) for t in si.make_qkv(6200, B, H, H, N, d))
    ref_c = eab.attention(q, k, v, causal=True)
    ref_n = eab.attention(q, k, v, causal=False)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for i in range(8):
        oc, lc = torch.full_like(q, float("nan")), torch.full((B, H, N), float("nan"), device=DEV)
        on, ln = torch.full_like(q, float("nan")), torch.full((B, H, N), float("nan"), device=DEV)
        torch.cuda.synchronize()
        eab.attn_fwd(q, k, v, oc, lc, True, d ** -0.5, s1)
        eab.attn_fwd(q, k, v, on, ln, False, d ** -0.5, s2)
        outs.append((oc, lc, on, ln))
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    for oc, lc, on, ln in outs:
        assert torch.equal(oc, ref_c[0]) and torch.equal(lc, ref_c[1])
        assert torch.equal(on, ref_n[0]) and torch.equal(ln, ref_n[1])

"""Runs one kernel of the library a few times on seeded inputs, for profilers.

    python -m exact_attention_ring_b200.profile_case fwd --B 4 --H 32 --N 2048 --d 128 --causal 1 --iters 3
    python -m exact_attention_ring_b200.profile_case decode --B 1 --H 32 --Hkv 8 --L 131072 --d 128 --iters 3
    python -m exact_attention_ring_b200.profile_case merge --B 2 --H 32 --N 8192 --d 128 --iters 3
    python -m exact_attention_ring_b200.profile_case ring --B 1 --H 32 --N 16384 --d 128 --world 8 --causal 1
    python -m exact_attention_ring_b200.profile_case bwd --B 4 --H 32 --N 2048 --d 128 --causal 1 --iters 3

Meant to be wrapped by ncu (one kernel, a few launches, inputs larger than L2
but a few GB at most). Prints the CUDA-event time of the last launch.
"""
import argparse
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import exact_attention_ring_b200 as eab  # noqa: E402
import seeded_inputs as si  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("kernel", choices=["fwd", "decode", "merge", "ring", "bwd"])
    ap.add_argument("--B", type=int, default=4)
    ap.add_argument("--H", type=int, default=32)
    ap.add_argument("--Hkv", type=int, default=0)
    ap.add_argument("--N", type=int, default=2048)
    ap.add_argument("--L", type=int, default=131072)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--causal", type=int, default=1)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--world", type=int, default=4, help="ring: virtual ranks emulated on this GPU")
    a = ap.parse_args()
    Hkv = a.Hkv or a.H
    dev = torch.device("cuda", 0)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if a.kernel == "fwd":
        q, k, v = (t.to(dev) for t in si.make_qkv(1001, a.B, a.H, Hkv, a.N, a.d))
        o = torch.empty_like(q)
        lse = torch.empty(a.B, a.H, a.N, device=dev)
        for _ in range(a.iters):
            start.record()
            eab.attn_fwd(q, k, v, o, lse, bool(a.causal), a.d ** -0.5)
            end.record()
        flops = 4.0 * a.B * a.H * a.N * a.N * a.d / (2 if a.causal else 1)
    elif a.kernel == "merge":
        # one merge step of a ring: rows = B*H*N, fp32 accumulator read and
        # written, fp32 block and the two LSE vectors read
        rows = a.B * a.H * a.N
        g = torch.Generator().manual_seed(1005)
        o_acc = torch.randn(rows, a.d, generator=g).to(dev)
        lse_acc = torch.randn(rows, generator=g).to(dev)
        o_blk = torch.randn(rows, a.d, generator=g).to(dev)
        lse_blk = torch.randn(rows, generator=g).to(dev)
        for _ in range(a.iters):
            start.record()
            eab.attn_merge(o_acc, lse_acc, o_blk, lse_blk)
            end.record()
        flops = rows * (a.d * (4 + 4 + 4) + 4 * 3)  # bytes for merge
    elif a.kernel == "bwd":
        # the three launches of attn_bwd (Delta, dK/dV, dQ) on the forward's O, LSE;
        # FLOPs counted as the five N x N x d products of the backward pass
        q, k, v = (t.to(dev) for t in si.make_qkv(1001, a.B, a.H, Hkv, a.N, a.d))
        do = si.make_dout(1002, a.B, a.H, a.N, a.d).to(dev)
        o, lse = eab.attention(q, k, v, bool(a.causal), a.d ** -0.5)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        delta = torch.empty_like(lse)
        for _ in range(a.iters):
            start.record()
            eab.attn_bwd(q, k, v, o, lse, do, delta, dq, dk, dv, bool(a.causal), a.d ** -0.5)
            end.record()
        flops = 10.0 * a.B * a.H * a.N * a.N * a.d / (2 if a.causal else 1)
    elif a.kernel == "ring":
        # every virtual rank's steps of the ring, one after another on this GPU:
        # the whole ring's attention and merge work (no exchange)
        q, k, v = (t.to(dev) for t in si.make_qkv(1001, a.B, a.H, Hkv, a.N, a.d))
        for _ in range(a.iters):
            start.record()
            eab.ring_attention_emulated(q, k, v, a.world, bool(a.causal), a.d ** -0.5)
            end.record()
        flops = 4.0 * a.B * a.H * a.N * a.N * a.d / (2 if a.causal else 1)
    else:
        q, k, v = (t.to(dev) for t in si.make_decode(1004, a.B, a.H, Hkv, a.L, a.d))
        S = eab.attn_decode_default_splits(a.B, a.H, Hkv, a.L)
        o_part = torch.empty(a.B, a.H, S, a.d, device=dev)
        lse_part = torch.empty(a.B, a.H, S, device=dev)
        for _ in range(a.iters):
            start.record()
            eab.attn_decode_splitkv(q, k, v, o_part, lse_part, S, a.d ** -0.5)
            end.record()
        flops = 2.0 * a.B * Hkv * a.L * a.d * 2  # bytes for decode
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    ms = start.elapsed_time(end)
    tensor = a.kernel in ("fwd", "ring", "bwd")
    unit = "TFLOPS" if tensor else "GB/s"
    val = flops / (ms * 1e-3) / (1e12 if tensor else 1e9)
    print(f"{a.kernel}: {ms:.4f} ms  {val:.1f} {unit}")


if __name__ == "__main__":
    main()

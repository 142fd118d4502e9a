"""Seeded synthetic inputs shared by the tests, the oracle checks and the bench.

This module only draws random numbers and names workload shapes. It holds no
attention arithmetic: both the CUDA path and the float64 oracle receive the
exact same host bytes from here, so any disagreement between them comes from
the computation and never from the inputs.

Recipe (the workloads of "1-Flash-Attention.md" on huajishe.fun, section
"问题分析": Q, K, V of shape (batch, heads, seq_len, head_dim)):
  * a CPU ``torch.Generator`` seeded with ``seed``;
  * ``randn`` in float32, drawn in the order q, k, v;
  * rounded to bfloat16 (round-to-nearest-even) by ``.to(torch.bfloat16)``;
  * the "large logits" variant multiplies the bf16 Q by 8, a power of two,
    so the scaled values are still exactly representable in bf16.
Layouts are contiguous row-major: q ``[B,Hq,N,d]``, k/v ``[B,Hkv,N,d]``;
decode q ``[B,Hq,d]`` with k/v ``[B,Hkv,L,d]``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


def _randn_bf16(gen: torch.Generator, shape, dtype=torch.bfloat16) -> torch.Tensor:
    # N(0,1) drawn in fp32, then rounded (RNE) to the input type
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(dtype)


def make_qkv(seed: int, B: int, Hq: int, Hkv: int, N: int, d: int, q_mult: float = 1.0,
             dtype=torch.bfloat16):
    """Prefill inputs: (q, k, v) as contiguous CPU tensors (bf16, or fp16)."""
    gen = torch.Generator().manual_seed(seed)
    q = _randn_bf16(gen, (B, Hq, N, d), dtype)
    k = _randn_bf16(gen, (B, Hkv, N, d), dtype)
    v = _randn_bf16(gen, (B, Hkv, N, d), dtype)
    if q_mult != 1.0:
        assert math.log2(q_mult).is_integer(), "q_mult must be a power of two (exact in bf16 and fp16)"
        q = (q.float() * q_mult).to(dtype)
    return q.contiguous(), k.contiguous(), v.contiguous()


def make_dout(seed: int, B: int, Hq: int, N: int, d: int, dtype=torch.bfloat16):
    """Output gradient for the backward pass: dO [B,Hq,N,d], N(0,1) rounded to
    the input type, from its own generator (seed independent of q, k, v)."""
    gen = torch.Generator().manual_seed(seed)
    return _randn_bf16(gen, (B, Hq, N, d), dtype).contiguous()


def make_decode(seed: int, B: int, Hq: int, Hkv: int, L: int, d: int, pin: bool = False, dtype=torch.bfloat16):
    """Single-query decode inputs: q [B,Hq,d], k/v [B,Hkv,L,d], CPU tensors (bf16, or fp16).

    Drawn in the order q, then k one batch entry at a time, then v likewise,
    so that a large cache never needs a full float32 copy on the host.
    """
    gen = torch.Generator().manual_seed(seed)
    q = _randn_bf16(gen, (B, Hq, d), dtype).contiguous()
    k = torch.empty(B, Hkv, L, d, dtype=dtype, pin_memory=pin)
    v = torch.empty(B, Hkv, L, d, dtype=dtype, pin_memory=pin)
    for t in (k, v):
        for b in range(B):
            t[b] = _randn_bf16(gen, (Hkv, L, d), dtype)
    return q, k, v


def make_signs(seed: int, d: int) -> torch.Tensor:
    """Random signs (+1 / -1, fp32 [d]) for the incoherent-processing rotation:
    the method draws them once and shares them between Q and K."""
    gen = torch.Generator().manual_seed(seed)
    return torch.where(torch.rand(d, generator=gen) < 0.5, -1.0, 1.0).to(torch.float32)


def with_outlier_channels(x: torch.Tensor, channels=((3, 20.0), (77, 15.0))) -> torch.Tensor:
    """x with a few head-dimension channels scaled up (the outlier features the
    FP8 rotation is meant for), rounded back to x's type."""
    xf = x.float().clone()
    for c, m in channels:
        if c < xf.shape[-1]:
            xf[..., c] *= m
    return xf.to(x.dtype).contiguous()


def sample_rows(seed: int, B: int, H: int, N: int, tile: int = 128, per_slice: int = 256,
                max_slices: int = 4):
    """Flat row indices ((b*H + h)*N + i) for sampled parity checks.

    Every sampled (b, h) slice contributes row 0, the last row, the rows on
    both sides of every tile boundary and ``per_slice`` random rows.
    """
    gen = torch.Generator().manual_seed(seed)
    nslices = B * H
    pick = torch.randperm(nslices, generator=gen)[: min(max_slices, nslices)].tolist()
    out = []
    for s in sorted(pick):
        rows = {0, N - 1}
        for t in range(tile, N, tile):
            rows.update({t - 1, t, min(t + 1, N - 1)})
        rnd = torch.randint(0, N, (per_slice,), generator=gen).tolist()
        rows.update(rnd)
        out.extend(s * N + i for i in sorted(rows))
    return torch.tensor(out, dtype=torch.int64)


@dataclass(frozen=True)
class PrefillShape:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    q_mult: float = 1.0
    seed: int = 1000

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def flops(self) -> float:
        f = 4.0 * self.B * self.Hq * self.N * self.N * self.d
        return f / 2 if self.causal else f


@dataclass(frozen=True)
class DecodeShape:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    d: int
    seed: int = 1004

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def kv_bytes(self) -> int:
        return 2 * self.B * self.Hkv * self.L * self.d * 2


# The five workload families (sizes as stated for the method's evaluation).
SINGLE_HEAD = PrefillShape("single-head B1 H1 N256 d64", 1, 1, 1, 256, 64, False, seed=1000)

LLAMA7B = [
    PrefillShape(f"llama7b B2 H32 N2048 d128 causal={c} qx{m:g}", 2, 32, 32, 2048, 128, c, m, 1001)
    for c in (True, False) for m in (1.0, 8.0)
]


def sweep_shapes():
    out = []
    idx = 0
    for d in (64, 128):
        for N in (512, 1024, 2048, 4096, 8192, 16384):
            for c in (True, False):
                out.append(PrefillShape(f"sweep d{d} N{N} causal={c}", 16384 // N, 2048 // d,
                                        2048 // d, N, d, c, seed=1002 * 100 + idx))
                idx += 1
    return out


GQA = [PrefillShape(f"gqa B1 Hq32 Hkv{h} N8192 d128 causal", 1, 32, h, 8192, 128, True, seed=1003)
       for h in (8, 1)]

DECODE = [DecodeShape(f"decode B{b} Hq32 Hkv8 L{L} d128", b, 32, 8, L, 128, seed=1004)
          for b in (1, 8) for L in (4096, 32768, 131072)]

"""Float64 CPU oracle for exact attention (ctypes wrapper over attn_oracle.cpp).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU
baseline leg may import this package; the product library never does. It
shares no code with the CUDA path. Inputs are torch CPU tensors (bf16, f32 or
f64); bf16 values are widened to double inside the C++ code.

Parity pins (tests/test_oracle_pins.py) tie every function here to facts the
pages and mathematics fix; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os

import torch

from .build import build_oracle, library_path

_lib = None
_DT = {torch.float64: 0, torch.bfloat16: 1, torch.float32: 2, torch.float16: 3}


def _load(plant: int = 0):
    global _lib
    if plant:
        return _bind(ctypes.CDLL(build_oracle(plant=plant)))
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            build_oracle()
        _lib = _bind(ctypes.CDLL(path))
    return _lib


def _bind(lib):
    P, I, D, L = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_int64
    lib.oracle_attention_rows.argtypes = [I, P, P, P, I, I, I, I, I, I, I, D, P, L, P, P, P, I]
    lib.oracle_attention_rows.restype = I
    lib.oracle_attention_blockwise_rows.argtypes = [I, P, P, P, I, I, I, I, I, I, I, D, I, P, L, P, P, I]
    lib.oracle_attention_blockwise_rows.restype = I
    lib.oracle_decode_partials.argtypes = [I, P, P, P, I, I, I, I, I, I, I, D, P, P, I]
    lib.oracle_decode_partials.restype = I
    lib.oracle_combine.argtypes = [P, P, I, I, I, I, P, P]
    lib.oracle_combine.restype = I
    lib.oracle_hardware_threads.restype = I
    lib.oracle_widen.argtypes = [I, P, L, P]
    lib.oracle_widen.restype = I
    lib.oracle_attention_backward.argtypes = [I, P, P, P, P, I, I, I, I, I, I, D, P, P, P, I]
    lib.oracle_attention_backward.restype = I
    lib.oracle_quant_fp8.argtypes = [I, P, I, I, I, I, P, P]
    lib.oracle_quant_fp8.restype = I
    lib.oracle_e4m3_decode.argtypes = [P, L, P]
    lib.oracle_e4m3_decode.restype = I
    lib.oracle_e4m3_encode.argtypes = [P, L, P]
    lib.oracle_e4m3_encode.restype = I
    lib.oracle_hadamard_rotate.argtypes = [P, P, L, I, P]
    lib.oracle_hadamard_rotate.restype = I
    return lib


def _ptr(t: torch.Tensor):
    return ctypes.c_void_p(t.data_ptr())


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (code {rc})")


def hardware_threads() -> int:
    return _load().oracle_hardware_threads()


def _prep(q, k, v):
    assert q.dtype == k.dtype == v.dtype and q.dtype in _DT
    return q.contiguous(), k.contiguous(), v.contiguous(), _DT[q.dtype]


def attention(q, k, v, causal: bool, scale: float, rows=None, nthreads: int = 0,
              want_probs: bool = False, plant: int = 0):
    """Direct definition. q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d].

    Returns (o, lse[, probs]) as float64. With ``rows`` (flat indices
    (b*Hq+h)*Nq+i) only those rows are computed: o [R,d], lse [R].
    """
    q, k, v, dt = _prep(q, k, v)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    full = rows is None
    if full:
        rows = torch.arange(B * Hq * Nq, dtype=torch.int64)
    rows = rows.to(torch.int64).contiguous()
    R = rows.numel()
    o = torch.empty(R, d, dtype=torch.float64)
    lse = torch.empty(R, dtype=torch.float64)
    probs = torch.empty(R, Nk, dtype=torch.float64) if want_probs else None
    rc = _load(plant).oracle_attention_rows(dt, _ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Nq, Nk, d,
                                            int(causal), float(scale), _ptr(rows), R, _ptr(o),
                                            _ptr(lse), _ptr(probs) if want_probs else None, nthreads)
    _check(rc, "attention")
    if full:
        o, lse = o.view(B, Hq, Nq, d), lse.view(B, Hq, Nq)
        if want_probs:
            probs = probs.view(B, Hq, Nq, Nk)
    return (o, lse, probs) if want_probs else (o, lse)


def attention_blockwise(q, k, v, causal: bool, scale: float, block_k: int, rows=None,
                        nthreads: int = 0, plant: int = 0):
    """The tiled online-softmax recurrence; same shapes and returns as attention()."""
    q, k, v, dt = _prep(q, k, v)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    full = rows is None
    if full:
        rows = torch.arange(B * Hq * Nq, dtype=torch.int64)
    rows = rows.to(torch.int64).contiguous()
    R = rows.numel()
    o = torch.empty(R, d, dtype=torch.float64)
    lse = torch.empty(R, dtype=torch.float64)
    rc = _load(plant).oracle_attention_blockwise_rows(dt, _ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Nq,
                                                      Nk, d, int(causal), float(scale), int(block_k),
                                                      _ptr(rows), R, _ptr(o), _ptr(lse), nthreads)
    _check(rc, "attention_blockwise")
    if full:
        return o.view(B, Hq, Nq, d), lse.view(B, Hq, Nq)
    return o, lse


def decode_partials(q, k, v, scale: float, num_splits: int, chunk: int, nthreads: int = 0,
                    plant: int = 0):
    """q [B,Hq,d], k/v [B,Hkv,L,d] -> o_part [B,Hq,S,d], lse_part [B,Hq,S] (float64)."""
    q, k, v, dt = _prep(q, k, v)
    B, Hq, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    o = torch.empty(B, Hq, num_splits, d, dtype=torch.float64)
    lse = torch.empty(B, Hq, num_splits, dtype=torch.float64)
    rc = _load(plant).oracle_decode_partials(dt, _ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, L, d,
                                             num_splits, chunk, float(scale), _ptr(o), _ptr(lse),
                                             nthreads)
    _check(rc, "decode_partials")
    return o, lse


def combine(o_part, lse_part, plant: int = 0):
    """o_part [B,Hq,S,d], lse_part [B,Hq,S] -> o [B,Hq,d], lse [B,Hq] (float64)."""
    o_part = o_part.to(torch.float64).contiguous()
    lse_part = lse_part.to(torch.float64).contiguous()
    B, Hq, S, d = o_part.shape
    o = torch.empty(B, Hq, d, dtype=torch.float64)
    lse = torch.empty(B, Hq, dtype=torch.float64)
    rc = _load(plant).oracle_combine(_ptr(o_part), _ptr(lse_part), B, Hq, S, d, _ptr(o), _ptr(lse))
    _check(rc, "combine")
    return o, lse


def decode(q, k, v, scale: float, rows=None, nthreads: int = 0):
    """Single-query decode by the direct definition: q [B,Hq,d] sees all L keys."""
    B, Hq, d = q.shape
    o, lse = attention(q.unsqueeze(2), k, v, False, scale, rows=rows, nthreads=nthreads)
    if rows is None:
        return o.view(B, Hq, d), lse.view(B, Hq)
    return o, lse


def widen(x):
    """The oracle's own widening of an input tensor (any of its input types) to
    float64, element by element (test hook for the format conversions)."""
    x = x.contiguous()
    n = x.numel()
    lib = _load()
    out = torch.empty(n, dtype=torch.float64)
    rc = lib.oracle_widen(_DT[x.dtype], _ptr(x), n, _ptr(out))
    _check(rc, "widen")
    return out.view(x.shape)


def attention_backward(q, k, v, dout, causal: bool, scale: float, nthreads: int = 0):
    """Gradients of sum(dout * O) for O = softmax(scale Q K^T) V (masked):
    returns (dq [B,Hq,N,d], dk [B,Hkv,N,d], dv [B,Hkv,N,d]) as float64."""
    q, k, v, dt = _prep(q, k, v)
    dout = dout.contiguous()
    assert dout.dtype == q.dtype and dout.shape == q.shape
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    dq = torch.empty(B, Hq, N, d, dtype=torch.float64)
    dk = torch.empty(B, Hkv, N, d, dtype=torch.float64)
    dv = torch.empty(B, Hkv, N, d, dtype=torch.float64)
    rc = _load().oracle_attention_backward(dt, _ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, Hq, Hkv, N, d,
                                           int(causal), float(scale), _ptr(dq), _ptr(dk), _ptr(dv), nthreads)
    _check(rc, "attention_backward")
    return dq, dk, dv


def e4m3_encode(x, plant: int = 0):
    """E4M3 codes (uint8) of a float32 tensor: nearest value, ties to even,
    saturated at +-448."""
    x = x.to(torch.float32).contiguous()
    out = torch.empty(x.shape, dtype=torch.uint8)
    _check(_load(plant).oracle_e4m3_encode(_ptr(x), x.numel(), _ptr(out)), "e4m3_encode")
    return out


def e4m3_decode(codes):
    """Values (float64) of E4M3 codes."""
    codes = codes.contiguous()
    assert codes.dtype == torch.uint8
    out = torch.empty(codes.shape, dtype=torch.float64)
    _check(_load().oracle_e4m3_decode(_ptr(codes), codes.numel(), _ptr(out)), "e4m3_decode")
    return out


def quant_fp8(x, per_plane: bool = False, plant: int = 0):
    """Block quantisation of x [..., N, d] (bf16, f32 or f16) to E4M3: returns
    (codes uint8 of x's shape, scales fp32 [..., ceil(N / 128)]), one scale per
    128-row block (per_plane: one per [N, d] plane, repeated per block)."""
    x = x.contiguous()
    *lead, N, d = x.shape
    planes = 1
    for n in lead:
        planes *= n
    nblk = (N + 127) // 128
    codes = torch.empty(x.shape, dtype=torch.uint8)
    scales = torch.empty(*lead, nblk, dtype=torch.float32)
    _check(_load(plant).oracle_quant_fp8(_DT[x.dtype], _ptr(x), planes, N, d, int(per_plane), _ptr(codes),
                                         _ptr(scales)), "quant_fp8")
    return codes, scales


def dequant_fp8(codes, scales):
    """float64 values codes stand for: e4m3 value x the scale of the row's block."""
    N = codes.shape[-2]
    rep = scales.to(torch.float64).repeat_interleave(128, dim=-1)[..., :N]
    return e4m3_decode(codes) * rep.unsqueeze(-1)


def hadamard_rotate(x, signs, plant: int = 0):
    """Incoherent-processing rotation of the rows of x [..., d] (fp32 result):
    y = H (signs o x) / sqrt(d), H the Sylvester Hadamard matrix, computed as
    the fast Walsh-Hadamard transform in fp32."""
    xf = x.to(torch.float32).contiguous()
    sg = signs.to(torch.float32).contiguous()
    d = xf.shape[-1]
    assert sg.shape == (d,)
    y = torch.empty_like(xf)
    _check(_load(plant).oracle_hadamard_rotate(_ptr(xf), _ptr(sg), xf.numel() // d, d, _ptr(y)), "hadamard_rotate")
    return y

"""ctypes binding of the C ABI in include/attn.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "_lib", "libattn_b200.so")

ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_CUDA, ATTN_ERR_TIMEOUT = range(5)


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_status_name(status)}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"exact_attention_ring_b200: CUDA library not built ({_LIB_PATH}); "
            "run `python exact_attention_ring_b200/build.py`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.attn_fwd.restype = I
    lib.attn_fwd_f32.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.attn_fwd_f32.restype = I
    lib.attn_fwd_f16.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.attn_fwd_f16.restype = I
    lib.attn_decode_splitkv_f16.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.attn_decode_splitkv_f16.restype = I
    lib.attn_combine_f16.argtypes = [P, P, P, P, I, I, I, I, P]
    lib.attn_combine_f16.restype = I
    lib.attn_decode_splitkv.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.attn_decode_splitkv.restype = I
    lib.attn_combine.argtypes = [P, P, P, P, I, I, I, I, P]
    lib.attn_combine.restype = I
    lib.attn_decode_default_splits.argtypes = [I, I, I, I]
    lib.attn_decode_default_splits.restype = I
    lib.attn_status_string.argtypes = [I]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_device_status.argtypes = [P]
    lib.attn_device_status.restype = I
    lib.attn_selftest_bounded_wait.argtypes = [I, P]
    lib.attn_selftest_bounded_wait.restype = I
    lib.attn_decode_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.attn_decode_noalloc.restype = I
    lib.attn_merge.argtypes = [P, P, P, P, P, ctypes.c_longlong, I, I, P]
    lib.attn_merge.restype = I
    lib.attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.attn_bwd.restype = I
    lib.attn_quant_fp8.argtypes = [P, P, P, I, I, I, I, I, P]
    lib.attn_quant_fp8.restype = I
    lib.attn_quant_fp8_rotate.argtypes = [P, P, P, P, I, I, I, P]
    lib.attn_quant_fp8_rotate.restype = I
    lib.attn_fwd_fp8.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.attn_fwd_fp8.restype = I
    return lib


_lib = _load()


def _status_name(status: int) -> str:
    return _lib.attn_status_string(int(status)).decode()


def attn_status_string(status: int) -> str:
    return _status_name(status)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(status: int, what: str):
    if status != ATTN_OK:
        raise AttnError(status, what)


def _need(t: torch.Tensor, dtype, name: str):
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")


# -------------------------------------------------------------- C ABI calls --

def _fwd(fn, name, dt, q, k, v, o, lse, causal, scale, stream):
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, dt, n)
    _need(lse, torch.float32, "lse")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape or o.shape != q.shape or lse.shape != (B, Hq, N):
        raise ValueError(f"{name}: inconsistent shapes")
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d, int(bool(causal)), float(scale),
              _stream(stream)), name)


def attn_fwd(q, k, v, o, lse, causal: bool, scale: float, stream=None):
    """q [B,Hq,N,d], k/v [B,Hkv,N,d], o [B,Hq,N,d] bf16; lse [B,Hq,N] fp32."""
    _fwd(_lib.attn_fwd, "attn_fwd", torch.bfloat16, q, k, v, o, lse, causal, scale, stream)


def attn_fwd_f16(q, k, v, o, lse, causal: bool, scale: float, stream=None):
    """attn_fwd for fp16 q, k, v and o."""
    _fwd(_lib.attn_fwd_f16, "attn_fwd_f16", torch.float16, q, k, v, o, lse, causal, scale, stream)


def attn_fwd_f32(q, k, v, o, lse, causal: bool, scale: float, stream=None):
    """attn_fwd with o [B,Hq,N,d] in fp32 (not rounded to bf16)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    _need(o, torch.float32, "o")
    _need(lse, torch.float32, "lse")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape or o.shape != q.shape or lse.shape != (B, Hq, N):
        raise ValueError("attn_fwd_f32: inconsistent shapes")
    _check(_lib.attn_fwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d, int(bool(causal)),
                             float(scale), _stream(stream)), "attn_fwd_f32")


def attn_bwd(q, k, v, o, lse, dout, delta, dq, dk, dv, causal: bool, scale: float, stream=None):
    """Gradients of attention: q, o, dout, dq [B,Hq,N,d] and k, v, dk, dv [B,Hkv,N,d]
    bf16; lse (from attn_fwd) and the workspace delta [B,Hq,N] fp32."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need(t, torch.bfloat16, n)
    _need(lse, torch.float32, "lse")
    _need(delta, torch.float32, "delta")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if (k.shape != (B, Hkv, N, d) or v.shape != k.shape or dk.shape != k.shape or dv.shape != k.shape
            or o.shape != q.shape or dout.shape != q.shape or dq.shape != q.shape
            or lse.shape != (B, Hq, N) or delta.shape != (B, Hq, N)):
        raise ValueError("attn_bwd: inconsistent shapes")
    _check(_lib.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(delta), _ptr(dq),
                         _ptr(dk), _ptr(dv), B, Hq, Hkv, N, d, int(bool(causal)), float(scale), _stream(stream)),
           "attn_bwd")


def attn_quant_fp8(x, codes, scales, per_plane: bool = False, transpose: bool = False, stream=None):
    """E4M3 block quantisation of x [..., N, d] bf16: codes uint8 [..., N, d]
    (transpose: [..., d, Np], Np = 128 * ceil(N / 128)), scales fp32
    [..., ceil(N / 128)]."""
    _need(x, torch.bfloat16, "x")
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.float32, "scales")
    *lead, N, d = x.shape
    planes = 1
    for n in lead:
        planes *= n
    nblk = -(-N // 128)
    want = (*lead, d, nblk * 128) if transpose else tuple(x.shape)
    if tuple(codes.shape) != want or tuple(scales.shape) != (*lead, nblk):
        raise ValueError("attn_quant_fp8: inconsistent shapes")
    _check(_lib.attn_quant_fp8(_ptr(x), _ptr(codes), _ptr(scales), planes, N, d, int(bool(per_plane)),
                               int(bool(transpose)), _stream(stream)), "attn_quant_fp8")


def attn_quant_fp8_rotate(x, signs, codes, scales, stream=None):
    """E4M3 block quantisation (per 128-row block, row-major codes) of x [..., N, d]
    bf16 after the incoherent-processing rotation y = H (signs o x) / sqrt(d);
    signs [d] fp32 of +1 / -1."""
    _need(x, torch.bfloat16, "x")
    _need(signs, torch.float32, "signs")
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.float32, "scales")
    *lead, N, d = x.shape
    planes = 1
    for n in lead:
        planes *= n
    if tuple(signs.shape) != (d,) or tuple(codes.shape) != tuple(x.shape) or \
            tuple(scales.shape) != (*lead, -(-N // 128)):
        raise ValueError("attn_quant_fp8_rotate: inconsistent shapes")
    _check(_lib.attn_quant_fp8_rotate(_ptr(x), _ptr(signs), _ptr(codes), _ptr(scales), planes, N, d,
                                      _stream(stream)), "attn_quant_fp8_rotate")


def attn_fwd_fp8(q8, k8, vt8, sq, sk, sv, o, lse, causal: bool, scale: float, stream=None):
    """q8 [B,Hq,N,128], k8 [B,Hkv,N,128], vt8 [B,Hkv,128,Np] E4M3 codes (uint8) with
    their scales; o [B,Hq,N,128] bf16, lse [B,Hq,N] fp32."""
    for t, n in ((q8, "q8"), (k8, "k8"), (vt8, "vt8")):
        _need(t, torch.uint8, n)
    for t, n in ((sq, "sq"), (sk, "sk"), (sv, "sv"), (lse, "lse")):
        _need(t, torch.float32, n)
    _need(o, torch.bfloat16, "o")
    B, Hq, N, d = q8.shape
    Hkv = k8.shape[1]
    nblk = -(-N // 128)
    if (k8.shape != (B, Hkv, N, d) or vt8.shape != (B, Hkv, d, nblk * 128) or sq.shape != (B, Hq, nblk)
            or sk.shape != (B, Hkv, nblk) or sv.shape != (B, Hkv, nblk) or o.shape != q8.shape
            or lse.shape != (B, Hq, N)):
        raise ValueError("attn_fwd_fp8: inconsistent shapes")
    _check(_lib.attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(vt8), _ptr(sq), _ptr(sk), _ptr(sv), _ptr(o), _ptr(lse),
                             B, Hq, Hkv, N, d, int(bool(causal)), float(scale), _stream(stream)), "attn_fwd_fp8")


def _dec(fn, name, dt, q, k, v, o_part, lse_part, num_splits, scale, stream):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, dt, n)
    _need(o_part, torch.float32, "o_part")
    _need(lse_part, torch.float32, "lse_part")
    B, Hq, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    S = int(num_splits)
    if k.shape != (B, Hkv, L, d) or v.shape != k.shape or o_part.shape != (B, Hq, S, d) \
            or lse_part.shape != (B, Hq, S):
        raise ValueError(f"{name}: inconsistent shapes")
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o_part), _ptr(lse_part), B, Hq, Hkv, L, d, S, float(scale),
              _stream(stream)), name)


def attn_decode_splitkv(q, k, v, o_part, lse_part, num_splits: int, scale: float, stream=None):
    """q [B,Hq,d], k/v [B,Hkv,L,d] bf16; o_part [B,Hq,S,d], lse_part [B,Hq,S] fp32."""
    _dec(_lib.attn_decode_splitkv, "attn_decode_splitkv", torch.bfloat16, q, k, v, o_part, lse_part, num_splits,
         scale, stream)


def attn_decode_splitkv_f16(q, k, v, o_part, lse_part, num_splits: int, scale: float, stream=None):
    """attn_decode_splitkv for fp16 q, k, v."""
    _dec(_lib.attn_decode_splitkv_f16, "attn_decode_splitkv_f16", torch.float16, q, k, v, o_part, lse_part,
         num_splits, scale, stream)


def _comb(fn, name, dt, o_part, lse_part, o, lse, stream):
    _need(o_part, torch.float32, "o_part")
    _need(lse_part, torch.float32, "lse_part")
    _need(o, dt, "o")
    _need(lse, torch.float32, "lse")
    B, Hq, S, d = o_part.shape
    if lse_part.shape != (B, Hq, S) or o.shape != (B, Hq, d) or lse.shape != (B, Hq):
        raise ValueError(f"{name}: inconsistent shapes")
    _check(fn(_ptr(o_part), _ptr(lse_part), _ptr(o), _ptr(lse), B, Hq, S, d, _stream(stream)), name)


def attn_combine(o_part, lse_part, o, lse, stream=None):
    """o_part [B,Hq,S,d], lse_part [B,Hq,S] fp32 -> o [B,Hq,d] bf16, lse [B,Hq] fp32."""
    _comb(_lib.attn_combine, "attn_combine", torch.bfloat16, o_part, lse_part, o, lse, stream)


def attn_combine_f16(o_part, lse_part, o, lse, stream=None):
    """attn_combine with o in fp16."""
    _comb(_lib.attn_combine_f16, "attn_combine_f16", torch.float16, o_part, lse_part, o, lse, stream)


def attn_merge(o_acc, lse_acc, o_blk, lse_blk, out=None, init=False, stream=None):
    """Folds one block's (o_blk fp32 [..., d], lse_blk fp32 [...]) into the running
    (o_acc fp32, lse_acc fp32) of the same shape; with `out` (bf16) the merged O
    goes there instead of into o_acc. Rows = lse_blk.numel()."""
    _need(o_acc, torch.float32, "o_acc")
    _need(lse_acc, torch.float32, "lse_acc")
    _need(o_blk, torch.float32, "o_blk")
    _need(lse_blk, torch.float32, "lse_blk")
    if out is not None:
        _need(out, torch.bfloat16, "out")
    d = o_blk.shape[-1]
    rows = lse_blk.numel()
    if (o_acc.shape != o_blk.shape or lse_acc.shape != lse_blk.shape or o_blk.numel() != rows * d
            or (out is not None and out.shape != o_blk.shape)):
        raise ValueError("attn_merge: inconsistent shapes")
    _check(_lib.attn_merge(_ptr(o_acc), _ptr(lse_acc), _ptr(o_blk), _ptr(lse_blk), _ptr(out), rows, d,
                           1 if init else 0, _stream(stream)), "attn_merge")


def attn_decode_default_splits(B: int, Hq: int, Hkv: int, L: int) -> int:
    return int(_lib.attn_decode_default_splits(B, Hq, Hkv, L))


def attn_device_status(stream=None) -> int:
    """Synchronises the stream, returns (and clears) the device-side status."""
    return int(_lib.attn_device_status(_stream(stream)))


def attn_selftest_bounded_wait(limit_us: int, stream=None):
    _check(_lib.attn_selftest_bounded_wait(int(limit_us), _stream(stream)), "attn_selftest_bounded_wait")


def decode_chunk(L: int, num_splits: int) -> int:
    """Keys per split used by attn_decode_splitkv: 128 * ceil(ceil(L / S) / 128)."""
    per = -(-L // num_splits)
    return -(-per // 128) * 128


# ------------------------------------------------------------- convenience --

def attention(q, k, v, causal: bool = False, scale: float | None = None, stream=None):
    """Allocates o, lse and runs attn_fwd (attn_fwd_f16 for fp16 inputs).
    Returns (o in the input type, lse fp32)."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], device=q.device, dtype=torch.float32)
    (attn_fwd_f16 if q.dtype == torch.float16 else attn_fwd)(q, k, v, o, lse, causal, scale, stream)
    return o, lse


def attention_backward(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None, stream=None):
    """Allocates dq, dk, dv (and the Delta workspace) and runs attn_bwd on the
    forward's (o, lse). Returns (dq, dk, dv) in bf16."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    delta = torch.empty(q.shape[:3], device=q.device, dtype=torch.float32)
    attn_bwd(q, k, v, o, lse, dout, delta, dq, dk, dv, causal, scale, stream)
    return dq, dk, dv


def quantize_fp8(x, per_plane: bool = False, transpose: bool = False, stream=None):
    """Allocates and fills (codes, scales) for attn_quant_fp8."""
    *lead, N, d = x.shape
    nblk = -(-N // 128)
    shape = (*lead, d, nblk * 128) if transpose else tuple(x.shape)
    codes = torch.empty(shape, device=x.device, dtype=torch.uint8)
    scales = torch.empty(*lead, nblk, device=x.device, dtype=torch.float32)
    attn_quant_fp8(x, codes, scales, per_plane, transpose, stream)
    return codes, scales


def quantize_fp8_rotated(x, signs, stream=None):
    """Allocates and fills (codes, scales) for attn_quant_fp8_rotate."""
    *lead, N, d = x.shape
    codes = torch.empty(tuple(x.shape), device=x.device, dtype=torch.uint8)
    scales = torch.empty(*lead, -(-N // 128), device=x.device, dtype=torch.float32)
    attn_quant_fp8_rotate(x, signs, codes, scales, stream)
    return codes, scales


def attention_fp8(q, k, v, causal: bool = False, scale: float | None = None, signs=None, stream=None):
    """FP8 forward from bf16 q, k, v: quantises Q and K per 128-row block and V
    per plane (transposed), then runs attn_fwd_fp8. With ``signs`` ([d] fp32 of
    +1 / -1, drawn by the caller) Q and K are rotated first (incoherent
    processing), which leaves Q K^T unchanged. Returns (o bf16, lse fp32)."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if signs is None:
        q8, sq = quantize_fp8(q, stream=stream)
        k8, sk = quantize_fp8(k, stream=stream)
    else:
        q8, sq = quantize_fp8_rotated(q, signs, stream=stream)
        k8, sk = quantize_fp8_rotated(k, signs, stream=stream)
    vt8, sv = quantize_fp8(v, per_plane=True, transpose=True, stream=stream)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], device=q.device, dtype=torch.float32)
    attn_fwd_fp8(q8, k8, vt8, sq, sk, sv, o, lse, causal, scale, stream)
    return o, lse


def decode(q, k, v, scale: float | None = None, num_splits: int | None = None, stream=None):
    """Split-KV decode plus combine (bf16 or fp16 inputs). q [B,Hq,d], k/v [B,Hkv,L,d] ->
    (o [B,Hq,d] in the input type, lse [B,Hq])."""
    B, Hq, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    S = num_splits or attn_decode_default_splits(B, Hq, Hkv, L)
    o_part = torch.empty(B, Hq, S, d, device=q.device, dtype=torch.float32)
    lse_part = torch.empty(B, Hq, S, device=q.device, dtype=torch.float32)
    f16 = q.dtype == torch.float16
    (attn_decode_splitkv_f16 if f16 else attn_decode_splitkv)(q, k, v, o_part, lse_part, S, scale, stream)
    o = torch.empty(B, Hq, d, device=q.device, dtype=q.dtype)
    lse = torch.empty(B, Hq, device=q.device, dtype=torch.float32)
    (attn_combine_f16 if f16 else attn_combine)(o_part, lse_part, o, lse, stream)
    return o, lse


def attn_decode_noalloc(q, k, v, o, lse, num_splits: int, scale: float, stream=None):
    """Decode plus combine with the partials in the library's fixed device array
    (no allocation anywhere). q [B,Hq,d], k/v [B,Hkv,L,d] bf16 -> o [B,Hq,d] bf16,
    lse [B,Hq] fp32. Needs B*Hq*num_splits*(d+1) <= 1,048,576."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, torch.bfloat16, n)
    _need(lse, torch.float32, "lse")
    B, Hq, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, L, d) or v.shape != k.shape or o.shape != (B, Hq, d) or lse.shape != (B, Hq):
        raise ValueError("attn_decode_noalloc: inconsistent shapes")
    _check(_lib.attn_decode_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, L, d,
                                    int(num_splits), float(scale), _stream(stream)), "attn_decode_noalloc")

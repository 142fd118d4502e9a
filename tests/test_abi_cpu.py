"""Host-side tests of the C ABI: no GPU needed, nothing is launched.

The library must load, export every entry point include/attn.h declares, and
reject bad arguments with the documented status before touching the device.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location("eab_build", os.path.join(ROOT, "exact_attention_ring_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    return ctypes.CDLL(build.build())


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(attn_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("attn_fwd", "attn_decode_splitkv", "attn_combine"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_names_match_the_abi():
    import exact_attention_ring_b200 as eab
    for n in declared_functions():
        assert hasattr(eab, n), n


def _fwd(lib, q=16, k=32, v=48, o=64, lse=80, B=1, Hq=2, Hkv=1, N=8, d=64, causal=0, scale=0.125):
    P = ctypes.c_void_p
    lib.attn_fwd.restype = ctypes.c_int
    return lib.attn_fwd(P(q), P(k), P(v), P(o), P(lse), B, Hq, Hkv, N, d, causal, ctypes.c_float(scale), None)


def _fwd32(lib, q=16, k=32, v=48, o=64, lse=80, B=1, Hq=2, Hkv=1, N=8, d=64, causal=0, scale=0.125):
    P = ctypes.c_void_p
    lib.attn_fwd_f32.restype = ctypes.c_int
    return lib.attn_fwd_f32(P(q), P(k), P(v), P(o), P(lse), B, Hq, Hkv, N, d, causal, ctypes.c_float(scale), None)


def _fwd16(lib, q=16, k=32, v=48, o=64, lse=80, B=1, Hq=2, Hkv=1, N=8, d=64, causal=0, scale=0.125):
    P = ctypes.c_void_p
    lib.attn_fwd_f16.restype = ctypes.c_int
    return lib.attn_fwd_f16(P(q), P(k), P(v), P(o), P(lse), B, Hq, Hkv, N, d, causal, ctypes.c_float(scale), None)


def _dec16(lib, q=16, k=32, v=48, op=64, lp=80, B=1, Hq=4, Hkv=2, L=100, d=128, S=4, scale=0.1):
    P = ctypes.c_void_p
    lib.attn_decode_splitkv_f16.restype = ctypes.c_int
    return lib.attn_decode_splitkv_f16(P(q), P(k), P(v), P(op), P(lp), B, Hq, Hkv, L, d, S, ctypes.c_float(scale),
                                       None)


def _comb16(lib, op=16, lp=32, o=48, lse=64, B=1, Hq=4, S=3, d=64):
    P = ctypes.c_void_p
    lib.attn_combine_f16.restype = ctypes.c_int
    return lib.attn_combine_f16(P(op), P(lp), P(o), P(lse), B, Hq, S, d, None)


def _dec(lib, q=16, k=32, v=48, op=64, lp=80, B=1, Hq=4, Hkv=2, L=100, d=128, S=4, scale=0.1):
    P = ctypes.c_void_p
    lib.attn_decode_splitkv.restype = ctypes.c_int
    return lib.attn_decode_splitkv(P(q), P(k), P(v), P(op), P(lp), B, Hq, Hkv, L, d, S, ctypes.c_float(scale), None)


def _comb(lib, op=16, lp=32, o=48, lse=64, B=1, Hq=4, S=3, d=64):
    P = ctypes.c_void_p
    lib.attn_combine.restype = ctypes.c_int
    return lib.attn_combine(P(op), P(lp), P(o), P(lse), B, Hq, S, d, None)


INVALID, UNSUPPORTED = 1, 2


@pytest.mark.parametrize("kw", [dict(q=0), dict(k=0), dict(v=0), dict(o=0), dict(lse=0), dict(q=17),
                                dict(o=24), dict(B=0), dict(Hq=0), dict(Hkv=0), dict(N=0), dict(Hq=3, Hkv=2),
                                dict(causal=2), dict(scale=0.0), dict(scale=-1.0), dict(scale=float("inf")),
                                dict(scale=float("nan"))])
def test_fwd_rejects_invalid(lib, kw):
    assert _fwd(lib, **kw) == INVALID


@pytest.mark.parametrize("kw", [dict(q=0), dict(o=0), dict(o=24), dict(N=0), dict(Hq=3, Hkv=2), dict(causal=2),
                                dict(scale=0.0)])
def test_fwd_f32_rejects_invalid(lib, kw):
    assert _fwd32(lib, **kw) == INVALID


def test_fwd_f32_rejects_unsupported_head_dim(lib):
    assert _fwd32(lib, d=96) == UNSUPPORTED


@pytest.mark.parametrize("d", [0, 8, 32, 96, 256])
def test_fwd_rejects_unsupported_head_dim(lib, d):
    assert _fwd(lib, d=d) == UNSUPPORTED


@pytest.mark.parametrize("kw", [dict(q=0), dict(op=0), dict(lp=8), dict(L=0), dict(S=0), dict(S=101),
                                dict(Hq=5, Hkv=2), dict(scale=0.0), dict(B=0)])
def test_decode_rejects_invalid(lib, kw):
    assert _dec(lib, **kw) == INVALID


def test_decode_rejects_unsupported_head_dim(lib):
    assert _dec(lib, d=80) == UNSUPPORTED


@pytest.mark.parametrize("kw", [dict(op=0), dict(lse=4), dict(B=0), dict(Hq=0), dict(S=0)])
def test_combine_rejects_invalid(lib, kw):
    assert _comb(lib, **kw) == INVALID


def test_combine_rejects_unsupported_head_dim(lib):
    assert _comb(lib, d=100) == UNSUPPORTED


def _merge(lib, oa=16, la=32, ob=48, lb=64, out=0, rows=8, d=128, init=0):
    P = ctypes.c_void_p
    lib.attn_merge.restype = ctypes.c_int
    lib.attn_merge.argtypes = [P, P, P, P, P, ctypes.c_longlong, ctypes.c_int, ctypes.c_int, P]
    return lib.attn_merge(P(oa), P(la), P(ob), P(lb), P(out) if out else None, rows, d, init, None)


@pytest.mark.parametrize("kw", [dict(oa=0), dict(la=0), dict(ob=0), dict(lb=0), dict(oa=20), dict(lb=36),
                                dict(out=40), dict(rows=0), dict(rows=-5), dict(rows=1 << 40)])
def test_merge_rejects_invalid(lib, kw):
    assert _merge(lib, **kw) == INVALID


@pytest.mark.parametrize("d", [0, 32, 96, 256])
def test_merge_rejects_unsupported_head_dim(lib, d):
    assert _merge(lib, d=d) == UNSUPPORTED


@pytest.mark.parametrize("kw", [dict(q=0), dict(o=24), dict(N=0), dict(Hq=3, Hkv=2), dict(causal=2), dict(scale=0.0)])
def test_fwd_f16_rejects_invalid(lib, kw):
    assert _fwd16(lib, **kw) == INVALID


@pytest.mark.parametrize("kw", [dict(q=0), dict(lp=8), dict(L=0), dict(S=0), dict(Hq=5, Hkv=2)])
def test_decode_f16_rejects_invalid(lib, kw):
    assert _dec16(lib, **kw) == INVALID


@pytest.mark.parametrize("kw", [dict(op=0), dict(lse=4), dict(S=0)])
def test_combine_f16_rejects_invalid(lib, kw):
    assert _comb16(lib, **kw) == INVALID


def test_f16_calls_reject_unsupported_head_dim(lib):
    assert _fwd16(lib, d=96) == UNSUPPORTED and _dec16(lib, d=80) == UNSUPPORTED and _comb16(lib, d=100) == UNSUPPORTED


def test_status_strings(lib):
    lib.attn_status_string.restype = ctypes.c_char_p
    names = [lib.attn_status_string(i).decode() for i in range(5)]
    assert names == ["ATTN_OK", "ATTN_ERR_INVALID_ARG", "ATTN_ERR_UNSUPPORTED", "ATTN_ERR_CUDA",
                     "ATTN_ERR_TIMEOUT"]
    assert lib.attn_status_string(99).decode() == "ATTN_ERR_UNKNOWN"


def test_selftest_rejects_bad_limit(lib):
    lib.attn_selftest_bounded_wait.restype = ctypes.c_int
    assert lib.attn_selftest_bounded_wait(0, None) == INVALID
    assert lib.attn_selftest_bounded_wait(2_000_000, None) == INVALID


def test_default_splits(lib):
    f = lib.attn_decode_default_splits
    f.restype = ctypes.c_int
    assert f(0, 32, 8, 100) == 0 and f(1, 30, 8, 100) == 0
    # groups of 4 query heads run the keys-as-rows decode, two blocks per SM (296
    # on B200). B=1, 8 KV heads: 8 blocks per split -> 37 splits = one wave of 296
    assert f(1, 32, 8, 32768) == 37
    assert f(1, 32, 8, 131072) == 37
    # B=8: 64 blocks per split; 9 splits = 576 blocks = 1.95 waves of 296
    assert f(8, 32, 8, 32768) == 9
    assert f(8, 32, 8, 131072) == 9
    # a group of 64 query heads runs the query-rows decode, one block per SM
    assert f(1, 64, 1, 1000) == 8
    assert f(1, 1, 1, 1) == 1
    for L in (1, 31, 257, 100000):
        s = f(2, 16, 4, L)
        assert 1 <= s <= -(-L // 128)


def test_decode_chunk_rule():
    from exact_attention_ring_b200 import decode_chunk
    assert decode_chunk(4096, 16) == 256
    assert decode_chunk(32768, 37) == 896
    assert decode_chunk(100, 64) == 128
    assert decode_chunk(1, 1) == 128
    assert decode_chunk(131072, 5) == 26240


def _bwd(lib, q=16, k=32, v=48, o=64, lse=80, do=96, delta=112, dq=128, dk=144, dv=160, B=1, Hq=2, Hkv=1,
         N=8, d=64, causal=0, scale=0.125):
    P = ctypes.c_void_p
    lib.attn_bwd.restype = ctypes.c_int
    return lib.attn_bwd(P(q), P(k), P(v), P(o), P(lse), P(do), P(delta), P(dq), P(dk), P(dv), B, Hq, Hkv, N, d,
                        causal, ctypes.c_float(scale), None)


@pytest.mark.parametrize("kw", [dict(q=0), dict(k=0), dict(v=0), dict(o=0), dict(lse=0), dict(do=0),
                                dict(delta=0), dict(dq=0), dict(dk=0), dict(dv=0), dict(dq=136), dict(lse=84),
                                dict(B=0), dict(N=0), dict(Hq=3, Hkv=2), dict(causal=2), dict(scale=0.0),
                                dict(scale=float("nan")), dict(B=2, Hq=40000, Hkv=40000),
                                dict(N=65535 * 128 + 1)])
def test_bwd_rejects_invalid(lib, kw):
    """Rejected before any device call; the last case is past the tile kernels'
    65535 tiles of 128 rows."""
    assert _bwd(lib, **kw) == INVALID


@pytest.mark.parametrize("d", [0, 32, 96, 256])
def test_bwd_rejects_unsupported_head_dim(lib, d):
    assert _bwd(lib, d=d) == UNSUPPORTED


def _quant8(lib, x=16, c=32, s=48, planes=2, N=100, d=128, per_plane=0, transpose=0):
    P = ctypes.c_void_p
    lib.attn_quant_fp8.restype = ctypes.c_int
    return lib.attn_quant_fp8(P(x), P(c), P(s), planes, N, d, per_plane, transpose, None)


def _fwd8(lib, q=16, k=32, v=48, sq=64, sk=80, sv=96, o=112, lse=128, B=1, Hq=2, Hkv=1, N=8, d=128, causal=0,
          scale=0.125):
    P = ctypes.c_void_p
    lib.attn_fwd_fp8.restype = ctypes.c_int
    return lib.attn_fwd_fp8(P(q), P(k), P(v), P(sq), P(sk), P(sv), P(o), P(lse), B, Hq, Hkv, N, d, causal,
                            ctypes.c_float(scale), None)


@pytest.mark.parametrize("kw", [dict(x=0), dict(c=0), dict(s=0), dict(c=40), dict(planes=0), dict(N=0),
                                dict(per_plane=2), dict(transpose=-1), dict(planes=70000)])
def test_quant_fp8_rejects_invalid(lib, kw):
    assert _quant8(lib, **kw) == INVALID


@pytest.mark.parametrize("d", [0, 32, 96, 256])
def test_quant_fp8_rejects_unsupported_head_dim(lib, d):
    assert _quant8(lib, d=d) == UNSUPPORTED


@pytest.mark.parametrize("kw", [dict(q=0), dict(v=0), dict(sv=0), dict(o=0), dict(lse=8), dict(N=0),
                                dict(Hq=3, Hkv=2), dict(causal=2), dict(scale=0.0), dict(B=2, Hq=40000, Hkv=40000)])
def test_fwd_fp8_rejects_invalid(lib, kw):
    assert _fwd8(lib, **kw) == INVALID


@pytest.mark.parametrize("d", [64, 96, 256])
def test_fwd_fp8_rejects_unsupported_head_dim(lib, d):
    assert _fwd8(lib, d=d) == UNSUPPORTED


def _rot8(lib, x=16, signs=32, c=48, s=64, planes=2, N=100, d=128):
    P = ctypes.c_void_p
    lib.attn_quant_fp8_rotate.restype = ctypes.c_int
    return lib.attn_quant_fp8_rotate(P(x), P(signs), P(c), P(s), planes, N, d, None)


@pytest.mark.parametrize("kw", [dict(x=0), dict(signs=0), dict(signs=36), dict(c=0), dict(s=0), dict(planes=0),
                                dict(N=0), dict(planes=70000)])
def test_quant_fp8_rotate_rejects_invalid(lib, kw):
    assert _rot8(lib, **kw) == INVALID


# The longest sequence a call takes is 2^31 - 256: the 256-row block and 128-key
# tile counts rounded up from it still fit an int. One row more is rejected
# before anything is launched.
TOO_LONG = 2**31 - 255


def test_sequence_longer_than_the_limit_is_rejected(lib):
    assert _fwd(lib, N=TOO_LONG) == INVALID
    assert _fwd32(lib, N=TOO_LONG) == INVALID
    assert _fwd16(lib, N=TOO_LONG) == INVALID
    assert _bwd(lib, N=TOO_LONG) == INVALID
    assert _dec(lib, L=TOO_LONG) == INVALID
    assert _dec16(lib, L=TOO_LONG) == INVALID
    assert _quant8(lib, N=TOO_LONG) == INVALID
    assert _rot8(lib, N=TOO_LONG) == INVALID
    assert _fwd8(lib, N=TOO_LONG) == INVALID
    f = lib.attn_decode_default_splits
    f.restype = ctypes.c_int
    assert f(1, 32, 8, TOO_LONG) == 0
    assert f(1, 32, 8, TOO_LONG - 1) > 0

"""attn_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers cannot hand the library a buffer for the split partials (their
device memory belongs to an engine's own pool, or they run as a plug-in that
must not allocate, or a cudaMalloc does not fit their latency budget). The
no-allocation entry point keeps the partials in a fixed array compiled into
the library. This test calls it through the C ABI (ctypes on the shared
library itself), twice in a row with different problems, and checks each
result against the existing attn_decode_splitkv + attn_combine pair on the
same inputs and against the float64 oracle, within the tolerances the other
parity tests use. It also checks that a problem larger than the fixed array,
or with more splits than the combine takes, is rejected before any launch.

The file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import oracle
import seeded_inputs as si
from attn_check import assert_attn_close

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import exact_attention_ring_b200 as eab  # noqa: E402

ATTN_OK, ATTN_ERR_INVALID_ARG = 0, 1
SCRATCH_FLOATS = 1 << 20


@pytest.fixture(scope="module")
def lib():
    lib = ctypes.CDLL(eab.library_path())
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.attn_decode_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.attn_decode_noalloc.restype = I
    return lib


def _noalloc(lib, q, k, v, S, scale):
    B, Hq, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    o = torch.empty(B, Hq, d, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(B, Hq, device="cuda", dtype=torch.float32)
    P = ctypes.c_void_p
    st = lib.attn_decode_noalloc(P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()), P(o.data_ptr()),
                                 P(lse.data_ptr()), B, Hq, Hkv, L, d, S, ctypes.c_float(scale),
                                 P(torch.cuda.current_stream().cuda_stream))
    return st, o, lse


def test_noalloc_matches_existing_entry_point_twice(lib):
    problems = [(9100, 2, 32, 8, 5000, 128), (9101, 1, 8, 2, 777, 64)]
    for seed, B, Hq, Hkv, L, d in problems:
        q, k, v = (t.cuda() for t in si.make_decode(seed, B, Hq, Hkv, L, d))
        S = eab.attn_decode_default_splits(B, Hq, Hkv, L)
        scale = d ** -0.5
        st, o, lse = _noalloc(lib, q, k, v, S, scale)
        assert st == ATTN_OK
        o_ref, lse_ref = eab.decode(q, k, v, scale, num_splits=S)
        torch.cuda.synchronize()
        assert eab.attn_device_status() == ATTN_OK
        assert_attn_close(o, lse, o_ref.double().cpu(), lse_ref.double().cpu(), f"noalloc B{B} L{L} d{d}")
        o_or, lse_or = oracle.decode(q.cpu(), k.cpu(), v.cpu(), scale)
        assert_attn_close(o, lse, o_or, lse_or, f"noalloc vs oracle B{B} L{L} d{d}")


def test_noalloc_rejects_problems_beyond_the_array(lib):
    B, Hq, Hkv, L, d = 1, 64, 8, 40000, 128
    q, k, v = (t.cuda() for t in si.make_decode(9200, B, Hq, Hkv, L, d))
    S = SCRATCH_FLOATS // (B * Hq * (d + 1)) + 1  # one split more than fits
    st, _, _ = _noalloc(lib, q, k, v, S, d ** -0.5)
    assert st == ATTN_ERR_INVALID_ARG
    st, _, _ = _noalloc(lib, q, k, v, S - 1, d ** -0.5)
    assert st == ATTN_OK
    torch.cuda.synchronize()


def test_noalloc_rejects_more_splits_than_the_combine_takes(lib):
    # 12001 splits of a 64-wide head fit the array (12001 * 65 floats) but not the
    # combine's 12000 per-split weights: rejected before the decode is enqueued
    B, Hq, Hkv, L, d = 1, 1, 1, 13000, 64
    q, k, v = (t.cuda() for t in si.make_decode(9300, B, Hq, Hkv, L, d))
    st, _, _ = _noalloc(lib, q, k, v, 12001, d ** -0.5)
    assert st == ATTN_ERR_INVALID_ARG
    st, o, lse = _noalloc(lib, q, k, v, 12000, d ** -0.5)
    assert st == ATTN_OK
    torch.cuda.synchronize()
    assert eab.attn_device_status() == ATTN_OK
    o_or, lse_or = oracle.decode(q.cpu(), k.cpu(), v.cpu(), d ** -0.5)
    assert_attn_close(o, lse, o_or, lse_or, "noalloc 12000 splits")


def test_noalloc_rejects_a_sequence_past_the_length_limit(lib):
    # L = 2^31 - 255, one key past the longest sequence any call takes: rejected
    # before anything is enqueued, so small buffers stand in for the key/value arrays
    q, k, v = (t.cuda() for t in si.make_decode(9400, 1, 1, 1, 128, 64))
    o = torch.empty(1, 1, 64, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(1, 1, device="cuda", dtype=torch.float32)
    P = ctypes.c_void_p
    st = lib.attn_decode_noalloc(P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()), P(o.data_ptr()),
                                 P(lse.data_ptr()), 1, 1, 1, 2**31 - 255, 64, 4, ctypes.c_float(0.125),
                                 P(torch.cuda.current_stream().cuda_stream))
    assert st == ATTN_ERR_INVALID_ARG

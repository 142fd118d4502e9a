"""Exact attention on B200 (sm_100a): prefill forward, split-KV decode, combine.

Thin Python binding over the C ABI of ``_lib/libattn_b200.so`` (declared in
``include/attn.h``). The binding only marshals arguments: every step of the
computation runs in the library's CUDA kernels. There is no CPU fallback; if
the library has not been built, importing this package raises.

Low-level calls (same names and arguments as the C ABI, with torch tensors in
place of pointers; ``stream`` defaults to torch's current stream):
    attn_fwd(q, k, v, o, lse, causal, scale)
    attn_decode_splitkv(q, k, v, o_part, lse_part, num_splits, scale)
    attn_combine(o_part, lse_part, o, lse)
Convenience wrappers that allocate the outputs with torch:
    attention(q, k, v, causal=False, scale=None) -> (o, lse)
    decode(q, k, v, scale=None, num_splits=None) -> (o, lse)
"""
from ._binding import (  # noqa: F401
    AttnError,
    attention,
    attn_combine,
    attn_decode_default_splits,
    attn_decode_noalloc,
    attn_decode_splitkv,
    attn_device_status,
    attn_fwd,
    attn_selftest_bounded_wait,
    attn_status_string,
    decode,
    decode_chunk,
    library_path,
)

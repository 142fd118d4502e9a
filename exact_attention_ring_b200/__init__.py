"""Exact attention on B200 (sm_100a): prefill forward, split-KV decode, combine,
ring attention, backward pass, FP8 forward.

Thin Python binding over the C ABI of ``_lib/libattn_b200.so`` (declared in
``include/attn.h``). The binding only marshals arguments: every step of the
computation runs in the library's CUDA kernels. There is no CPU fallback; if
the library has not been built, importing this package raises.

Low-level calls (same names and arguments as the C ABI, with torch tensors in
place of pointers; ``stream`` defaults to torch's current stream):
    attn_fwd(q, k, v, o, lse, causal, scale)
    attn_fwd_f32(q, k, v, o, lse, causal, scale)   (o in fp32)
    attn_fwd_f16, attn_decode_splitkv_f16, attn_combine_f16   (fp16 inputs)
    attn_decode_splitkv(q, k, v, o_part, lse_part, num_splits, scale)
    attn_combine(o_part, lse_part, o, lse)
    attn_merge(o_acc, lse_acc, o_blk, lse_blk, out=None, init=False)
    attn_bwd(q, k, v, o, lse, dout, delta, dq, dk, dv, causal, scale)   (gradients)
    attn_quant_fp8(x, codes, scales, per_plane=False, transpose=False)  (E4M3 block quantisation)
    attn_quant_fp8_rotate(x, signs, codes, scales)  (the same after incoherent processing)
    attn_fwd_fp8(q8, k8, vt8, sq, sk, sv, o, lse, causal, scale)        (forward on E4M3 codes)
Ring attention (context parallelism, ``ring.py``): each rank attends its query
shard to every key/value shard as the shards travel around the ring of ranks,
merging with attn_merge:
    ring_attention(q, k, v, causal=False, scale=None, group=None) -> (o, lse)
Convenience wrappers that allocate the outputs with torch:
    attention(q, k, v, causal=False, scale=None) -> (o, lse)
    decode(q, k, v, scale=None, num_splits=None) -> (o, lse)
    attention_backward(q, k, v, o, lse, dout, causal=False, scale=None) -> (dq, dk, dv)
    quantize_fp8(x, per_plane=False, transpose=False) -> (codes, scales)
    attention_fp8(q, k, v, causal=False, scale=None, signs=None) -> (o, lse)
"""
from ._binding import (  # noqa: F401
    AttnError,
    attention,
    attention_backward,
    attention_fp8,
    attn_bwd,
    attn_combine,
    attn_combine_f16,
    attn_decode_default_splits,
    attn_decode_noalloc,
    attn_decode_splitkv,
    attn_decode_splitkv_f16,
    attn_device_status,
    attn_fwd,
    attn_fwd_f16,
    attn_fwd_f32,
    attn_fwd_fp8,
    attn_merge,
    attn_quant_fp8,
    attn_quant_fp8_rotate,
    attn_selftest_bounded_wait,
    attn_status_string,
    decode,
    decode_chunk,
    library_path,
    quantize_fp8,
    quantize_fp8_rotated,
)
from .ring import ring_attention, ring_attention_emulated, ring_schedule  # noqa: F401,E402

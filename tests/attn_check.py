"""Shared tolerance checks for the GPU-vs-oracle parity tests.

Bounds for bf16 inputs with fp32 accumulation: O max-abs <= 2e-2, O relative
RMS error (||O_gpu - O_ref||_2 / ||O_ref||_2) <= 5e-3, |LSE_gpu - LSE_ref| <= 1e-3.
"""
import torch

O_MAX_ABS = 2e-2
O_REL_RMS = 5e-3
LSE_ABS = 1e-3


def errors(o_gpu, lse_gpu, o_ref, lse_ref):
    o = o_gpu.detach().double().cpu().reshape(o_ref.shape)
    l = lse_gpu.detach().double().cpu().reshape(lse_ref.shape)
    diff = o - o_ref
    max_abs = diff.abs().max().item() if diff.numel() else 0.0
    ref_norm = o_ref.norm().item()
    rel_rms = diff.norm().item() / ref_norm if ref_norm > 0 else diff.norm().item()
    lse_abs = (l - lse_ref).abs().max().item() if l.numel() else 0.0
    return max_abs, rel_rms, lse_abs


def assert_attn_close(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    assert torch.isfinite(o_gpu).all() and torch.isfinite(lse_gpu).all(), f"{what}: non-finite output"
    max_abs, rel_rms, lse_abs = errors(o_gpu, lse_gpu, o_ref, lse_ref)
    assert max_abs <= O_MAX_ABS and rel_rms <= O_REL_RMS and lse_abs <= LSE_ABS, (
        f"{what}: max_abs={max_abs:.3e} rel_rms={rel_rms:.3e} lse_abs={lse_abs:.3e}")
    return max_abs, rel_rms, lse_abs

"""B200-native fused attention forward (FlashAttention-2 style) behind a C ABI.

``fa_fwd`` and friends (see include/fa.h) are exported by ``libfa.so``, a
hand-written sm_100a library (TMA, mbarrier pipelines, tcgen05 MMAs into
TMEM).  This package is the thin Python binding: it marshals torch tensors
(device memory and streams) into the C call.  No step of the computation runs
in Python or PyTorch, and there is no fallback path.
"""
from __future__ import annotations

from ._lib import (FA_BF16, FA_FP16, FaError, fa_check_status, fa_fwd, fa_fwd_noalloc, fa_last_timeout_site,
                   fa_num_units, fa_selftest_timeout, fa_status_string, fa_version, load)

__all__ = [
    "FA_BF16", "FA_FP16", "FaError", "fa_check_status", "fa_fwd", "fa_fwd_noalloc", "fa_last_timeout_site",
    "fa_num_units", "fa_selftest_timeout", "fa_status_string", "fa_version", "flash_attention_forward", "load",
]


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float16:
        return FA_FP16
    if t.dtype == torch.bfloat16:
        return FA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float16 or bfloat16")


def flash_attention_forward(q, k, v, scale: float, causal: bool = False, out=None, lse=None, stream=None):
    """O, LSE for contiguous BHSD CUDA tensors ``q, k, v`` ([B, H, S, D], fp16/bf16).

    ``scale`` is required (commonly 1/sqrt(D)).  ``out``/``lse`` may be given
    to reuse buffers.  Launches on ``stream`` (default: torch's current
    stream) and returns without synchronising.
    """
    import torch
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must all be [B, H, S, D] with the same shape")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous BHSD")
    B, H, S, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    if out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous():
        raise ValueError("out must be a contiguous tensor like q")
    if lse.shape != (B, H, S) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [B, H, S] tensor")
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    st = fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H, S, D,
                float(scale), int(bool(causal)), _dtype_code(q), int(stream.cuda_stream))
    if st != 0:
        raise FaError(st)
    return out, lse

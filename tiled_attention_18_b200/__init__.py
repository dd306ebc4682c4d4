"""B200-native fused attention (FlashAttention-2 style) behind a C ABI.

The entries of include/fa.h (forward and backward passes, their mask,
dropout, strided and combined variants, and the sequence-parallel helpers)
are exported by ``libfa.so``, a hand-written sm_100a library (TMA, mbarrier
pipelines, tcgen05 MMAs into TMEM).  This package is the thin Python binding:
it marshals torch tensors (device memory and streams) into the C calls.  No
step of the computation runs in Python or PyTorch, and there is no fallback
path: a missing library raises.  ``sequence_parallel`` orders the library's
calls and torch.distributed's communication for a sequence split across
ranks.
"""
from __future__ import annotations

from ._lib import (FA_BF16, FA_FP16, FaError, fa_accumulate, fa_backward, fa_bwd, fa_bwd_dropout, fa_bwd_ex,
                   fa_bwd_mask, fa_bwd_workspace_size, fa_check_status, fa_forward, fa_fwd, fa_fwd_dropout, fa_fwd_ex,
                   fa_fwd_mask, fa_fwd_noalloc, fa_last_cuda_error, fa_last_timeout_site, fa_merge_finalize,
                   fa_merge_partial, fa_num_units, fa_selftest_timeout, fa_status_string, fa_version, load)

__all__ = [
    "FA_BF16", "FA_FP16", "FaError", "fa_accumulate", "fa_backward", "fa_bwd", "fa_bwd_dropout", "fa_bwd_ex",
    "fa_bwd_mask", "fa_bwd_workspace_size", "fa_check_status", "fa_forward", "fa_fwd", "fa_fwd_dropout", "fa_fwd_ex",
    "fa_fwd_mask", "fa_fwd_noalloc", "fa_last_cuda_error", "fa_last_timeout_site", "fa_merge_finalize",
    "fa_merge_partial", "fa_num_units", "fa_selftest_timeout", "fa_status_string", "fa_version", "flash_attention_backward",
    "flash_attention_forward", "load",
]


_DTYPE_CODES = None


def _dtype_code(t) -> int:
    global _DTYPE_CODES
    if _DTYPE_CODES is None:
        import torch
        _DTYPE_CODES = {torch.float16: FA_FP16, torch.bfloat16: FA_BF16}
    code = _DTYPE_CODES.get(t.dtype)
    if code is None:
        raise TypeError(f"unsupported dtype {t.dtype}; expected float16 or bfloat16")
    return code


def _current_stream_handle(device) -> int:
    """The raw handle of torch's current stream on ``device`` (a plain int, without
    building a torch Stream object on every call when torch exposes it)."""
    import torch
    raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    if raw is not None:
        return int(raw(device.index if device.index is not None else torch.cuda.current_device()))
    return int(torch.cuda.current_stream(device).cuda_stream)


def _mask_stride(mask, B, H, Sq, Sk):
    """(b, h, row) element strides of a [B|1, H|1, Sq, Sk] uint8/bool CUDA mask (0 broadcasts)."""
    if mask.dim() != 4 or tuple(mask.shape[2:]) != (Sq, Sk) or mask.shape[0] not in (1, B) or \
            mask.shape[1] not in (1, H):
        raise ValueError("mask must be [B|1, H|1, Sq, Sk]")
    if mask.element_size() != 1 or not mask.is_cuda or (mask.stride(3) != 1 and Sk > 1):
        raise ValueError("mask must be a uint8/bool CUDA tensor with contiguous keys")
    return (mask.stride(0) if mask.shape[0] > 1 else 0, mask.stride(1) if mask.shape[1] > 1 else 0, mask.stride(2))


def flash_attention_forward(q, k, v, scale: float, causal: bool = False, out=None, lse=None, stream=None,
                            dropout_p: float = 0.0, seed: int = 0, offset: int = 0, mask=None, block_n: int = 0,
                            q_tiles: int = 0):
    """O, LSE for CUDA tensors ``q`` [B, H, Sq, D] and ``k, v`` [B, H, Sk, D] (fp16/bf16).

    The tensors may be any strided views whose last dimension is contiguous
    (for example ``x.transpose(1, 2)`` of a [B, S, H, D] tensor); b, h and s
    strides must be multiples of 8 elements.  With ``causal`` query i sees
    keys j <= i + Sk - Sq (requires Sq <= Sk).  ``scale`` is required
    (commonly 1/sqrt(D)).  ``out`` (like ``q``, any such strides) and ``lse``
    (contiguous float32 [B, H, Sq]) may be given to reuse buffers; by default
    ``out`` takes ``q``'s memory layout.  Launches on ``stream`` (default:
    torch's current stream) and returns without synchronising.

    ``dropout_p`` > 0 applies attention dropout after the softmax (the keep
    decisions are fixed by ``seed`` and ``offset``, which
    flash_attention_backward must be given too).  ``mask`` (a uint8/bool CUDA
    tensor [B|1, H|1, Sq, Sk], nonzero = attend, keys contiguous, row stride a
    multiple of 16 and >= Sk) restricts the keys each query sees.  Mask,
    dropout, strides and Sq != Sk combine freely (fa_forward).  ``block_n``
    (64 or 128 keys per key tile) and ``q_tiles`` (1 or 2 query tiles of 128
    rows per work unit) set the tiling by hand (0 = automatic; D = 64/128,
    without mask or dropout).
    """
    import torch
    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape:
        raise ValueError("q must be [B, H, Sq, D] and k, v [B, H, Sk, D]")
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    if k.shape[0] != B or k.shape[1] != H or k.shape[3] != D:
        raise ValueError("k and v must share q's B, H and D")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.stride(3) != 1 and D > 1:
            raise ValueError(f"{name} must be contiguous in its last dimension")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    if out.shape != q.shape or out.dtype != q.dtype or out.stride(3) != 1:
        raise ValueError("out must be like q, contiguous in its last dimension")
    if lse.shape != (B, H, Sq) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [B, H, Sq] tensor")
    st = _current_stream_handle(q.device) if stream is None else int(stream.cuda_stream)
    dt = _dtype_code(q)
    if dropout_p != 0.0 or mask is not None or block_n or q_tiles:
        rc = fa_forward(st, q=q.data_ptr(), k=k.data_ptr(), v=v.data_ptr(), o=out.data_ptr(), lse=lse.data_ptr(),
                        B=B, H=H, Sq=Sq, Sk=Sk, D=D, q_stride=q.stride()[:3], k_stride=k.stride()[:3],
                        v_stride=v.stride()[:3], o_stride=out.stride()[:3],
                        mask=mask.data_ptr() if mask is not None else None,
                        mask_stride=_mask_stride(mask, B, H, Sq, Sk) if mask is not None else None,
                        dropout_p=float(dropout_p), seed=seed, offset=offset, scale=float(scale),
                        causal=int(bool(causal)), dtype=dt, block_n=int(block_n), q_tiles=int(q_tiles))
        if rc != 0:
            raise FaError(rc, "fa_forward")
        return out, lse
    if Sq == Sk and all(t.is_contiguous() for t in (q, k, v, out)):
        rc = fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H, Sq, D,
                    float(scale), int(bool(causal)), dt, st)
    else:
        rc = fa_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H, Sq, Sk, D,
                       q.stride()[:3], k.stride()[:3], v.stride()[:3], out.stride()[:3], float(scale),
                       int(bool(causal)), dt, st)
    if rc != 0:
        raise FaError(rc)
    return out, lse


def flash_attention_backward(q, k, v, o, lse, dout, scale: float, causal: bool = False, deterministic: bool = False,
                             dq=None, dk=None, dv=None, workspace=None, stream=None, dropout_p: float = 0.0,
                             seed: int = 0, offset: int = 0, mask=None):
    """dQ, dK, dV for CUDA tensors q, o, dout [B, H, Sq, D] and k, v [B, H, Sk, D]
    (lse [B, H, Sq] fp32 from the forward call).  The tensors may be strided
    views contiguous in their last dimension (fa_bwd_ex), like the forward's;
    the gradients take the layouts of q, k, v unless given.  The
    workspace (fa_bwd_workspace_size bytes) is allocated with torch unless
    given.  Launches on ``stream`` (default: torch's current stream) and
    returns without synchronising.  ``dropout_p``, ``seed``, ``offset`` and
    ``mask`` must be those of the forward call (fa_backward when a mask or
    dropout is given)."""
    import torch
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        if not (t.is_cuda and t.dtype == q.dtype and (t.stride(3) == 1 or D == 1)):
            raise ValueError(f"{name} must be a CUDA tensor of q's dtype, contiguous in its last dimension")
    if o.shape != q.shape or dout.shape != q.shape or k.shape != (B, H, Sk, D) or v.shape != k.shape:
        raise ValueError("q, o, dout must be [B, H, Sq, D] and k, v [B, H, Sk, D]")
    if lse.shape != (B, H, Sq) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [B, H, Sq] tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    nbytes = fa_bwd_workspace_size(B, H, Sq, D)
    if nbytes < 0:
        raise FaError(nbytes, "fa_bwd_workspace_size")
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    sid = _current_stream_handle(q.device) if stream is None else int(stream.cuda_stream)
    tensors = (q, k, v, o, dout, dq, dk, dv)
    if dropout_p != 0.0 or mask is not None:
        names = ("q", "k", "v", "o", "dout", "dq", "dk", "dv")
        rc = fa_backward(sid, **{n: t.data_ptr() for n, t in zip(names, tensors)},
                         lse=lse.data_ptr(), workspace=workspace.data_ptr(), workspace_bytes=workspace.numel(),
                         B=B, H=H, Sq=Sq, Sk=Sk, D=D,
                         **{("do" if n == "dout" else n) + "_stride": t.stride()[:3] for n, t in zip(names, tensors)},
                         mask=mask.data_ptr() if mask is not None else None,
                         mask_stride=_mask_stride(mask, B, H, Sq, Sk) if mask is not None else None,
                         dropout_p=float(dropout_p), seed=seed, offset=offset, scale=float(scale),
                         causal=int(bool(causal)), deterministic=int(bool(deterministic)), dtype=_dtype_code(q))
        if rc != 0:
            raise FaError(rc, "fa_backward")
        return dq, dk, dv
    if not all(t.is_contiguous() for t in tensors):
        rc = fa_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                       dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(), workspace.numel(), B, H, Sq,
                       Sk, D, *(t.stride()[:3] for t in tensors), float(scale), int(bool(causal)),
                       int(bool(deterministic)), _dtype_code(q), sid)
        if rc != 0:
            raise FaError(rc, "fa_bwd_ex")
        return dq, dk, dv
    if dropout_p != 0.0:
        rc = fa_bwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(), workspace.numel(), B, H,
                            Sq, Sk, D, float(scale), int(bool(causal)), float(dropout_p), int(seed), int(offset),
                            int(bool(deterministic)), _dtype_code(q), sid)
        if rc != 0:
            raise FaError(rc, "fa_bwd_dropout")
        return dq, dk, dv
    rc = fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(), workspace.numel(), B, H, Sq, Sk, D,
                float(scale), int(bool(causal)), int(bool(deterministic)), _dtype_code(q), sid)
    if rc != 0:
        raise FaError(rc, "fa_bwd")
    return dq, dk, dv


from .autograd import attention  # noqa: E402  (the differentiable operation over the two calls above)

__all__.append("attention")

"""Shared helpers for the GPU parity tests (test infrastructure)."""
from __future__ import annotations

import numpy as np
import torch

import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import LSE_TOL, O_TOL


def half_ulp(x: np.ndarray, dtype: str) -> np.ndarray:
    """Half the spacing of the 16-bit format at |x| (the best possible rounding error)."""
    mant_bits = 10 if dtype == "fp16" else 7
    min_exp = -14 if dtype == "fp16" else -126
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, np.finfo(np.float64).tiny)))
    e = np.maximum(e, min_exp)
    return 0.5 * np.exp2(e - mant_bits)


def run_fa(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float, causal: bool):
    """Copy CPU inputs to the GPU, run fa_fwd through the C ABI, return CPU (O, LSE)."""
    dq, dk, dv = (t.to("cuda") for t in (q, k, v))
    o = torch.full_like(dq, float("nan"))
    lse = torch.full(dq.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    fa.flash_attention_forward(dq, dk, dv, scale, causal, out=o, lse=lse)
    st = fa.fa_check_status(torch.cuda.current_stream().cuda_stream)
    assert st == 0, f"device status {st} ({fa.fa_status_string(st)}), site {fa.fa_last_timeout_site():#x}"
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def compare(o_gpu: torch.Tensor, lse_gpu: torch.Tensor, o_ref: np.ndarray, lse_ref: np.ndarray, dtype: str):
    """Check the stated tolerances.  Returns a dict of error figures.

    O: max |O_gpu - O_ref| <= tol (2e-3 fp16, 1e-2 bf16) on every element whose
    own rounding floor (half an ulp of the dtype at O_ref) is below tol; where
    the format cannot represent O_ref to within tol, the GPU value must be one of
    the two representable neighbours (error <= 1 ulp).  LSE: max abs <= 1e-3.
    """
    tol = O_TOL[dtype]
    og = o_gpu.to(torch.float64).numpy()
    err = np.abs(og - o_ref)
    floor = half_ulp(o_ref, dtype)
    representable = floor < tol
    assert np.all(np.isfinite(og)), "non-finite output"
    max_err = float(err.max()) if err.size else 0.0
    max_err_repr = float(err[representable].max()) if representable.any() else 0.0
    n_floor = int((~representable).sum())
    assert max_err_repr <= tol, f"max |dO| {max_err_repr:.3g} > {tol} (dtype {dtype})"
    if n_floor:
        assert float((err[~representable] / (2 * floor[~representable])).max()) <= 1.0 + 1e-9
    lg = lse_gpu.to(torch.float64).numpy()
    assert np.all(np.isfinite(lg)), "non-finite LSE"
    lse_err = float(np.abs(lg - lse_ref).max()) if lg.size else 0.0
    assert lse_err <= LSE_TOL, f"max |dLSE| {lse_err:.3g} > {LSE_TOL}"
    return {"max_abs_o": max_err, "max_abs_o_representable": max_err_repr, "n_below_floor": n_floor,
            "max_abs_lse": lse_err}


def run_fa_ex(q, k, v, scale: float, causal: bool, layouts=("bhsd", "bhsd", "bhsd", "bhsd"), o_pad: int = 0):
    """fa_fwd_ex through the C ABI on CPU BHSD inputs placed on the GPU in the
    given layouts (q, k, v, o: "bhsd" | "bshd").  ``o_pad`` > 0 writes O into a
    view of a wider NaN-filled buffer (rows o_pad elements apart from the next
    row's start beyond D) and checks that the gaps stay NaN.
    Returns CPU (O contiguous BHSD, LSE)."""
    from tiled_attention_18_b200.workloads import to_layout
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    dq, dk, dv = (to_layout(t, lay).to("cuda") if lay == "bhsd" else
                  t.transpose(1, 2).contiguous().to("cuda").transpose(1, 2)
                  for t, lay in zip((q, k, v), layouts[:3]))
    if o_pad:
        if layouts[3] == "bhsd":
            buf = torch.full((B, H, Sq, D + o_pad), float("nan"), dtype=q.dtype, device="cuda")
            o = buf[..., :D]
        else:
            buf = torch.full((B, Sq, H, D + o_pad), float("nan"), dtype=q.dtype, device="cuda")
            o = buf[..., :D].transpose(1, 2)
    else:
        shape = (B, H, Sq, D) if layouts[3] == "bhsd" else (B, Sq, H, D)
        buf = torch.full(shape, float("nan"), dtype=q.dtype, device="cuda")
        o = buf if layouts[3] == "bhsd" else buf.transpose(1, 2)
    lse = torch.full((B, H, Sq), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    dt = fa.FA_BF16 if q.dtype == torch.bfloat16 else fa.FA_FP16
    rc = fa.fa_fwd_ex(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, Sq, Sk, D,
                      dq.stride()[:3], dk.stride()[:3], dv.stride()[:3], o.stride()[:3], scale, int(causal), dt, st)
    assert rc == 0, f"fa_fwd_ex returned {rc} ({fa.fa_status_string(rc)})"
    s = fa.fa_check_status(st)
    assert s == 0, f"device status {s} ({fa.fa_status_string(s)}), site {fa.fa_last_timeout_site():#x}"
    torch.cuda.synchronize()
    if o_pad:
        assert torch.isnan(buf[..., D:]).all(), "fa_fwd_ex wrote outside O's view"
    return o.contiguous().cpu(), lse.cpu()


UNIT_ROUNDOFF = {"fp16": 2.0 ** -11, "bf16": 2.0 ** -8}
# Half the spacing of the subnormal numbers: below the smallest normal value
# (2^-14 for fp16) rounding is absolute, at most this much.
SUBNORMAL_HALF_SPACING = {"fp16": 2.0 ** -25, "bf16": 2.0 ** -134}
# |dX - dX_ref| <= BWD_TOL_C * (u * mag_dX + eta * (abs_dX + 1)) element by
# element, u the unit roundoff (the largest relative error of one rounding to
# nearest).  dV: the weights are rounded once before P^T dO (at most u of
# mag_dV) and the result once (u |dV| <= u mag_dV).  dQ, dK: dS is rounded
# once (u P |dP - Delta|), Delta comes from the forward O whose error is at
# most 2u sum_k P |v| per element (both inside the oracle's magnitude term
# a_i), and the result is rounded once.  Below the smallest normal value a
# rounding is absolute, at most eta: eta times the sum of the other operand's
# absolute values per rounded factor, plus eta for the output.  fp32
# accumulation and the approximate exp2 add orders of magnitude less, so the
# total stays below 2 units.
BWD_TOL_C = 2.0


def _abs_sums(q, k, dout, scale, causal):
    """Per element of dQ, dK, dV: the sums of |k_j|, |q_i|, |dO_i| over the
    (query, key) pairs that contribute to it (times scale for dQ, dK)."""
    qa, ka, ga = (np.abs(t.to(torch.float64).numpy()) for t in (q, k, dout))
    Sq, Sk = qa.shape[2], ka.shape[2]
    sc = float(np.float32(scale))
    if not causal:
        return (sc * np.broadcast_to(ka.sum(axis=2, keepdims=True), qa.shape),
                sc * np.broadcast_to(qa.sum(axis=2, keepdims=True), ka.shape),
                np.broadcast_to(ga.sum(axis=2, keepdims=True), ka.shape))
    off = Sk - Sq
    kpre = np.cumsum(ka, axis=2)                       # keys 0..j
    n_vis = np.clip(np.arange(Sq) + off + 1, 0, Sk)    # keys seen by query i
    abs_dq = np.zeros(qa.shape)
    has = n_vis > 0
    abs_dq[:, :, has] = kpre[:, :, n_vis[has] - 1]
    qsuf = np.cumsum(qa[:, :, ::-1], axis=2)[:, :, ::-1]  # queries i..Sq-1
    gsuf = np.cumsum(ga[:, :, ::-1], axis=2)[:, :, ::-1]
    first = np.clip(np.arange(Sk) - off, 0, Sq)        # first query that sees key j
    abs_dk = np.zeros(ka.shape)
    abs_dv = np.zeros(ka.shape)
    ok = first < Sq
    abs_dk[:, :, ok] = qsuf[:, :, first[ok]]
    abs_dv[:, :, ok] = gsuf[:, :, first[ok]]
    return sc * abs_dq, sc * abs_dk, abs_dv


def run_fa_bwd(q, k, v, dout, scale: float, causal: bool, deterministic: bool = False):
    """Forward (fa_fwd_ex) then backward (fa_bwd) through the C ABI on CPU
    contiguous inputs; returns CPU (dQ, dK, dV, O, LSE)."""
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    dq_, dk_, dv_, ddo = (t.to("cuda") for t in (q, k, v, dout))
    o = torch.empty_like(dq_)
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    dt = fa.FA_BF16 if q.dtype == torch.bfloat16 else fa.FA_FP16
    rc = fa.fa_fwd_ex(dq_.data_ptr(), dk_.data_ptr(), dv_.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, Sq, Sk, D,
                      None, None, None, None, scale, int(causal), dt, st)
    assert rc == 0, rc
    gq = torch.full_like(dq_, float("nan"))
    gk = torch.full_like(dk_, float("nan"))
    gv = torch.full_like(dv_, float("nan"))
    ws_bytes = fa.fa_bwd_workspace_size(B, H, Sq, D)
    ws = torch.full((max(ws_bytes, 1),), 0xAB, dtype=torch.uint8, device="cuda")  # garbage on entry
    rc = fa.fa_bwd(dq_.data_ptr(), dk_.data_ptr(), dv_.data_ptr(), o.data_ptr(), ddo.data_ptr(), lse.data_ptr(),
                   gq.data_ptr(), gk.data_ptr(), gv.data_ptr(), ws.data_ptr(), ws_bytes, B, H, Sq, Sk, D, scale,
                   int(causal), int(deterministic), dt, st)
    assert rc == 0, f"fa_bwd returned {rc} ({fa.fa_status_string(rc)})"
    s = fa.fa_check_status(st)
    assert s == 0, f"device status {s} ({fa.fa_status_string(s)}), site {fa.fa_last_timeout_site():#x}"
    torch.cuda.synchronize()
    return gq.cpu(), gk.cpu(), gv.cpu(), o.cpu(), lse.cpu()


def compare_bwd(grads, refs, mags, dtype: str, q, k, dout, scale: float, causal: bool, c: float = BWD_TOL_C):
    """Element-wise bound c * (u * mag + eta * (abs + 1)) for dQ, dK, dV (c =
    BWD_TOL_C by default).  Returns the largest error as a multiple of that
    bound's unit for each gradient."""
    u = UNIT_ROUNDOFF[dtype]
    eta = SUBNORMAL_HALF_SPACING[dtype]
    abss = _abs_sums(q, k, dout, scale, causal)
    out = {}
    for name, g, r, m, a in zip(("dq", "dk", "dv"), grads, refs, mags, abss):
        gg = g.to(torch.float64).numpy()
        assert np.all(np.isfinite(gg)), f"non-finite {name}"
        err = np.abs(gg - r)
        unit = u * m + eta * (a + 1.0) + 1e-300
        worst = float((err / unit).max()) if err.size else 0.0
        assert worst <= c, f"{name}: error {worst:.3g} x bound unit > {c} (max abs {err.max():.3g})"
        out[name] = worst
    return out

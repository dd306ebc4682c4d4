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

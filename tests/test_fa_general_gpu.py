"""GPU parity of fa_fwd_ex (through the C ABI): Sq != Sk with and without the
bottom-right causal mask, and strided layouts read and written in place,
against the fp64 CPU oracle; bitwise agreement with fa_fwd where the two
compute the same thing."""
import numpy as np
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import (GENERAL_WORKLOADS, make_cross_inputs, make_inputs, sample_rows,
                                               softmax_scale, workload_inputs)

from gpu_helpers import compare, run_fa, run_fa_ex

pytestmark = pytest.mark.gpu

CROSS = [
    # (B, H, Sq, Sk, D)
    (1, 1, 1, 1, 64), (1, 2, 1, 300, 128), (2, 3, 77, 1000, 64), (1, 2, 300, 77, 128), (2, 2, 129, 1, 64),
    (1, 2, 100, 356, 64), (1, 2, 129, 700, 128), (1, 1, 256, 257, 64), (1, 3, 640, 1000, 64),
    (1, 1, 257, 128, 128), (1, 2, 513, 1100, 128),
]


@pytest.mark.parametrize("shape", CROSS, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_cross_shapes_match_oracle(shape, dtype, causal):
    B, H, Sq, Sk, D = shape
    if causal and Sq > Sk:
        pytest.skip("causal needs Sq <= Sk (checked on the host)")
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, dtype, seed=Sq * 7 + Sk)
    scale = softmax_scale(D)
    o, lse = run_fa_ex(q, k, v, scale, causal)
    o_ref, lse_ref = oracle.attn_fwd_gen(q, k, v, scale, causal, dtype)
    compare(o, lse, o_ref, lse_ref, dtype)


@pytest.mark.parametrize("layouts", [("bshd",) * 4, ("bshd", "bhsd", "bshd", "bhsd"), ("bhsd", "bshd", "bshd", "bshd")],
                         ids=["all-bshd", "mixed1", "mixed2"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("D", [64, 128])
def test_strided_layouts_match_oracle_and_contiguous(layouts, causal, D):
    B, H, Sq, Sk = 2, 3, 300, 433
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, "bf16", seed=D + int(causal))
    scale = softmax_scale(D)
    o, lse = run_fa_ex(q, k, v, scale, causal, layouts=layouts)
    o_ref, lse_ref = oracle.attn_fwd_gen(q, k, v, scale, causal, "bf16")
    compare(o, lse, o_ref, lse_ref, "bf16")
    # the layout changes only the addressing: bitwise the contiguous result
    o2, lse2 = run_fa_ex(q, k, v, scale, causal)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_packed_qkv_and_padded_output():
    """Q, K, V as slices of one packed [B, S, 3, H, D] buffer; O written into a
    [B, H, S, D + 64] buffer whose padding must stay untouched."""
    B, H, S, D = 2, 4, 777, 64
    q, k, v = make_inputs(B, H, S, D, "fp16", seed=31)
    packed = torch.stack([t.transpose(1, 2) for t in (q, k, v)], dim=2).contiguous().cuda()  # [B,S,3,H,D]
    dq, dk, dv = (packed[:, :, i].transpose(1, 2) for i in range(3))
    buf = torch.full((B, H, S, D + 64), float("nan"), dtype=torch.float16, device="cuda")
    o = buf[..., :D]
    lse = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    for causal in (0, 1):
        rc = fa.fa_fwd_ex(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, S, S, D,
                          dq.stride()[:3], dk.stride()[:3], dv.stride()[:3], o.stride()[:3], 0.125, causal,
                          fa.FA_FP16, st)
        assert rc == 0
        assert fa.fa_check_status(st) == 0
        o_ref, lse_ref = run_fa(q, k, v, 0.125, bool(causal))
        assert torch.equal(o.cpu(), o_ref) and torch.equal(lse.cpu(), lse_ref)
        assert torch.isnan(buf[..., D:]).all()


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_fa_fwd_ex_equals_fa_fwd_bitwise(causal):
    q, k, v = make_inputs(2, 5, 1000, 128, "bf16", seed=3)
    a = run_fa(q, k, v, 0.09, causal)
    b = run_fa_ex(q, k, v, 0.09, causal)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_zero_query_closed_form_with_offset(causal, dtype):
    B, H, Sq, Sk, D = 1, 2, 700, 2500, 64
    _, k, v = make_cross_inputs(B, H, Sq, Sk, D, dtype, seed=12)
    q = torch.zeros((B, H, Sq, D), dtype=k.dtype)
    o, lse = run_fa_ex(q, k, v, 0.125, causal)
    vd = v.to(torch.float64).numpy()
    off = Sk - Sq
    if causal:
        n = np.arange(1, Sq + 1, dtype=np.float64) + off
        ref = (np.cumsum(vd, axis=2) / np.arange(1, Sk + 1, dtype=np.float64)[None, None, :, None])[:, :, off:]
        ref_lse = np.broadcast_to(np.log(n), (B, H, Sq))
    else:
        ref = np.broadcast_to(vd.mean(axis=2, keepdims=True), (B, H, Sq, D))
        ref_lse = np.full((B, H, Sq), np.log(Sk))
    compare(o, lse, ref, ref_lse, dtype)


@pytest.mark.parametrize("name", ["sdxl_xattn", "bert_large"])
def test_general_workload_full_compare(name):
    w = GENERAL_WORKLOADS[name]
    q, k, v = workload_inputs(w)
    o, lse = run_fa_ex(q, k, v, w.scale, w.causal, layouts=(w.layout,) * 4)
    o_ref, lse_ref = oracle.attn_fwd_gen(q, k, v, w.scale, w.causal, w.dtype)
    print(name, compare(o, lse, o_ref, lse_ref, w.dtype))


def test_prefill_cached_sampled_rows():
    w = GENERAL_WORKLOADS["prefill_cached"]
    q, k, v = workload_inputs(w)
    o, lse = run_fa_ex(q, k, v, w.scale, w.causal)
    bh, rows = sample_rows(w.B, w.H, w.S, n_random=768, edge=2)
    o_ref, lse_ref = oracle.attn_rows_gen(q, k, v, w.scale, w.causal, w.dtype, bh, rows)
    og = o.reshape(w.B * w.H, w.S, w.D)[torch.from_numpy(bh), torch.from_numpy(rows)]
    lg = lse.reshape(w.B * w.H, w.S)[torch.from_numpy(bh), torch.from_numpy(rows)]
    print(compare(og, lg, o_ref, lse_ref, w.dtype))
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()

"""GPU parity of fa_bwd (through the C ABI) against the fp64 backward oracle.

The forward outputs O and LSE come from the GPU forward pass (the backward
pass's normal input); dQ, dK, dV are compared with the oracle's exact
gradients element by element within BWD_TOL_C * (u * mag + eta * (abs + 1))
(gpu_helpers), where mag is the oracle's absolute-value sum of the terms of
each element and eta * abs covers fp16 subnormals.  Larger
runs add the identities sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i.
"""
import numpy as np
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import make_cross_inputs, make_inputs, softmax_scale

from gpu_helpers import BWD_TOL_C, UNIT_ROUNDOFF, compare_bwd, run_fa_bwd

pytestmark = pytest.mark.gpu


def _dout(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    t = torch.randn(shape, generator=g, dtype=torch.float32)
    return t.to(torch.float16 if dtype == "fp16" else torch.bfloat16)


SHAPES = [
    # (B, H, Sq, Sk, D)
    (1, 1, 1, 1, 64), (1, 2, 17, 17, 128), (1, 1, 128, 128, 64), (1, 2, 129, 129, 128), (2, 1, 255, 255, 64),
    (1, 2, 300, 300, 128), (1, 1, 513, 513, 64), (1, 2, 77, 300, 128), (1, 1, 300, 77, 64), (2, 2, 200, 456, 64),
    (1, 1, 640, 1000, 128),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_bwd_small_shapes_match_oracle(shape, dtype, causal):
    B, H, Sq, Sk, D = shape
    if causal and Sq > Sk:
        pytest.skip("causal needs Sq <= Sk")
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, dtype, seed=Sq + 5 * Sk + D)
    dout = _dout(q.shape, dtype, seed=Sq * 3 + Sk)
    scale = softmax_scale(D)
    gq, gk, gv, _, _ = run_fa_bwd(q, k, v, dout, scale, causal)
    dq, dk, dv, mq, mk, mv = oracle.attn_bwd(q, k, v, dout, scale, causal, dtype, magnitudes=True)
    r = compare_bwd((gq, gk, gv), (dq, dk, dv), (mq, mk, mv), dtype, q, k, dout, scale, causal)
    print(shape, dtype, causal, r)


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_bwd_ops_transformer_example_full(causal):
    """The ops-transformer worked example's shape (B=2, H=12, S=2048, D=64, fp16)."""
    q, k, v = make_inputs(2, 12, 2048, 64, "fp16", seed=0)
    dout = _dout(q.shape, "fp16", seed=100)
    scale = softmax_scale(64)
    gq, gk, gv, _, _ = run_fa_bwd(q, k, v, dout, scale, causal)
    dq, dk, dv, mq, mk, mv = oracle.attn_bwd(q, k, v, dout, scale, causal, "fp16", magnitudes=True)
    print(compare_bwd((gq, gk, gv), (dq, dk, dv), (mq, mk, mv), "fp16", q, k, dout, scale, causal))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_bwd_long_sequence_identities(causal):
    """S = 8192, D = 128, bf16: every gradient finite, sum_j dK_j = 0 and
    sum_j dV_j = sum_i dO_i per head, and two runs agree on dK, dV bitwise."""
    B, H, S, D = 1, 4, 8192, 128
    q, k, v = make_inputs(B, H, S, D, "bf16", qk_mult=2.0, seed=3)
    dout = _dout(q.shape, "bf16", seed=4)
    gq, gk, gv, _, _ = run_fa_bwd(q, k, v, dout, softmax_scale(D), causal)
    for g in (gq, gk, gv):
        assert torch.isfinite(g).all()
    u = UNIT_ROUNDOFF["bf16"]
    gk64, gv64 = gk.to(torch.float64), gv.to(torch.float64)
    # each dK_j is rounded once (u/2 relative): the column sum vanishes to within that
    assert torch.all(gk64.sum(dim=2).abs() <= BWD_TOL_C * u * gk64.abs().sum(dim=2) + 1e-6)
    ref_v = dout.to(torch.float64).sum(dim=2)
    assert torch.all((gv64.sum(dim=2) - ref_v).abs() <= BWD_TOL_C * u * gv64.abs().sum(dim=2) + 1e-6)
    gq2, gk2, gv2, _, _ = run_fa_bwd(q, k, v, dout, softmax_scale(D), causal)
    assert torch.equal(gk, gk2) and torch.equal(gv, gv2)


def test_bwd_zero_queries_zero_key_gradients():
    k = torch.randn(1, 2, 100, 64).to(torch.float16).cuda()
    dk = torch.full_like(k, float("nan"))
    dv = torch.full_like(k, float("nan"))
    st = torch.cuda.current_stream().cuda_stream
    rc = fa.fa_bwd(0, k.data_ptr(), k.data_ptr(), 0, 0, 0, 0, dk.data_ptr(), dv.data_ptr(), 0, 0, 1, 2, 0, 100, 64,
                   0.125, 0, 0, fa.FA_FP16, st)
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.all(dk == 0) and torch.all(dv == 0)


def test_bwd_rejects_small_workspace():
    q = torch.zeros((1, 1, 128, 64), dtype=torch.float16, device="cuda")
    lse = torch.zeros((1, 1, 128), dtype=torch.float32, device="cuda")
    need = fa.fa_bwd_workspace_size(1, 1, 128, 64)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    p = q.data_ptr()
    assert fa.fa_bwd(p, p, p, p, p, lse.data_ptr(), p, p, p, ws.data_ptr(), need - 1, 1, 1, 128, 128, 64, 0.125, 0,
                     0, fa.FA_FP16, st) == -13
    assert fa.fa_bwd(p, p, p, p, p, lse.data_ptr(), p, p, p, ws.data_ptr() + 16, need, 1, 1, 128, 128, 64, 0.125, 0,
                     0, fa.FA_FP16, st) == -13


@pytest.mark.parametrize("shape", [(1, 2, 300, 300, 128), (2, 2, 200, 456, 64), (1, 1, 513, 513, 64),
                                   (1, 2, 640, 1000, 128)], ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_bwd_deterministic_mode_matches_oracle(shape, causal):
    B, H, Sq, Sk, D = shape
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, "bf16", seed=Sq + Sk)
    dout = _dout(q.shape, "bf16", seed=Sq)
    scale = softmax_scale(D)
    gq, gk, gv, _, _ = run_fa_bwd(q, k, v, dout, scale, causal, deterministic=True)
    dq, dk, dv, mq, mk, mv = oracle.attn_bwd(q, k, v, dout, scale, causal, "bf16", magnitudes=True)
    print(compare_bwd((gq, gk, gv), (dq, dk, dv), (mq, mk, mv), "bf16", q, k, dout, scale, causal))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_bwd_deterministic_mode_is_bitwise_repeatable(D, causal):
    """S = 4096 (32 key tiles per head): dQ, dK, dV identical over three runs."""
    q, k, v = make_inputs(1, 6, 4096, D, "bf16", seed=21)
    dout = _dout(q.shape, "bf16", seed=22)
    runs = [run_fa_bwd(q, k, v, dout, softmax_scale(D), causal, deterministic=True)[:3] for _ in range(3)]
    for r in runs[1:]:
        for a, b in zip(r, runs[0]):
            assert torch.equal(a, b)
    # and it agrees with the atomic mode to rounding (same products, another order of dQ sums)
    ga = run_fa_bwd(q, k, v, dout, softmax_scale(D), causal)[:3]
    assert torch.equal(ga[1], runs[0][1]) and torch.equal(ga[2], runs[0][2])
    assert torch.allclose(ga[0].float(), runs[0][0].float(), rtol=2e-2, atol=2e-3)

"""Attention dropout on the GPU (fa_fwd_dropout, fa_bwd_dropout) against the
fp64 oracle: the keep decisions bit-exact (read back through V = identity),
p = 0 equal to the kernels without dropout, the forward within the forward's
tolerances (scaled by 1 / (1 - p)), the backward within the gradient bound,
and sampled rows of a full-size run."""
import numpy as np
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import LSE_TOL, O_TOL, make_cross_inputs, make_inputs, softmax_scale

from gpu_helpers import compare_bwd, half_ulp

pytestmark = pytest.mark.gpu


def p8_of(p):
    return int(np.floor(p * 256 + 0.5))


def run_fwd_dropout(q, k, v, scale, causal, p, seed, offset):
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    o, lse = fa.flash_attention_forward(dq, dk, dv, scale, causal, dropout_p=p, seed=seed, offset=offset)
    st = fa.fa_check_status(torch.cuda.current_stream().cuda_stream)
    assert st == 0, fa.fa_status_string(st)
    return o.cpu(), lse.cpu()


def check_o(o_gpu, lse_gpu, o_ref, lse_ref, dtype, p):
    """The forward's tolerance scaled by the kept weights' factor 1 / (1 - p)."""
    zs = 256.0 / (256.0 - p8_of(p))
    tol = O_TOL[dtype] * zs
    og = o_gpu.double().numpy()
    err = np.abs(og - o_ref)
    rep = half_ulp(o_ref, dtype) < tol
    assert np.all(np.isfinite(og))
    assert err[rep].max() <= tol, f"max |dO| {err[rep].max():.3g} > {tol:.3g}"
    if (~rep).any():
        assert (err[~rep] / (2 * half_ulp(o_ref, dtype)[~rep])).max() <= 1 + 1e-9
    lerr = np.abs(lse_gpu.double().numpy() - lse_ref).max()
    assert lerr <= LSE_TOL
    return float(err.max()), float(lerr)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_keep_decisions_bit_exact(D, dtype):
    """V = identity over D keys: O[i, j] = P_ij z_ij / l, zero exactly where the
    weight was dropped; the zero pattern must equal the oracle's keep mask."""
    B, H, S = 2, 3, D
    q, k, _ = make_inputs(B, H, S, D, dtype, seed=D)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    v = torch.eye(D, dtype=tdt).expand(B, H, D, D).contiguous()
    for p, seed, offset in ((0.1, 1, 0), (0.5, 0xDEADBEEFCAFE, 7), (0.9, 42, 123456)):
        o, _ = run_fwd_dropout(q, k, v, softmax_scale(D), False, p, seed, offset)
        keep = oracle.dropout_keep_mask(B * H, S, S, p8_of(p), seed, offset).reshape(B, H, S, S)
        got = (o.float().numpy() != 0).astype(np.uint8)
        assert np.array_equal(got, keep), f"p={p}: {int((got != keep).sum())} decisions differ"


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("fp16", 64), ("fp16", 128), ("bf16", 64)])
@pytest.mark.parametrize("p", [0.1, 0.5])
def test_forward_matches_oracle(causal, dtype, D, p):
    q, k, v = make_inputs(1, 3, 300, D, dtype, seed=5)
    scale = softmax_scale(D)
    o, lse = run_fwd_dropout(q, k, v, scale, causal, p, seed=77, offset=3)
    o_ref, lse_ref = oracle.attn_fwd_dropout(q, k, v, scale, causal, dtype, p8_of(p), 77, 3)
    print(check_o(o, lse, o_ref, lse_ref, dtype, p))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_forward_cross_shapes(causal):
    q, k, v = make_cross_inputs(2, 2, 200, 333, 128, "bf16", seed=9)
    o, lse = run_fwd_dropout(q, k, v, 0.09, causal, 0.2, seed=5, offset=1)
    o_ref, lse_ref = oracle.attn_fwd_dropout(q, k, v, 0.09, causal, "bf16", p8_of(0.2), 5, 1)
    check_o(o, lse, o_ref, lse_ref, "bf16", 0.2)


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("fp16", 64)])
def test_p0_equals_no_dropout_bitwise(dtype, D):
    q, k, v = make_cross_inputs(1, 2, 257, 300, D, dtype, seed=2)
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    o0, l0 = fa.flash_attention_forward(dq, dk, dv, 0.1, True)
    o1 = torch.empty_like(o0)
    l1 = torch.empty_like(l0)
    dt = fa.FA_BF16 if dtype == "bf16" else fa.FA_FP16
    st = torch.cuda.current_stream().cuda_stream
    assert fa.fa_fwd_dropout(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), o1.data_ptr(), l1.data_ptr(), 1, 2, 257, 300,
                             D, 0.1, 1, 0.0, 3, 4, dt, st) == 0
    torch.cuda.synchronize()
    assert torch.equal(o0, o1) and torch.equal(l0, l1)
    # the LSE never depends on the dropout
    _, l2 = fa.flash_attention_forward(dq, dk, dv, 0.1, True, dropout_p=0.3, seed=3, offset=4)
    torch.cuda.synchronize()
    assert torch.equal(l0, l2)


def run_bwd_dropout(q, k, v, dout, scale, causal, p, seed, offset, deterministic=False):
    dq_, dk_, dv_, ddo = (t.cuda() for t in (q, k, v, dout))
    o, lse = fa.flash_attention_forward(dq_, dk_, dv_, scale, causal, dropout_p=p, seed=seed, offset=offset)
    gq, gk, gv = fa.flash_attention_backward(dq_, dk_, dv_, o, lse, ddo, scale, causal, deterministic=deterministic,
                                             dropout_p=p, seed=seed, offset=offset)
    st = fa.fa_check_status(torch.cuda.current_stream().cuda_stream)
    assert st == 0, fa.fa_status_string(st)
    return gq.cpu(), gk.cpu(), gv.cpu()


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("fp16", 128), ("bf16", 64), ("fp16", 64)])
@pytest.mark.parametrize("shape", [(1, 2, 300, 300), (2, 1, 190, 257)], ids=["square", "cross"])
def test_backward_matches_oracle(causal, dtype, D, shape):
    B, H, Sq, Sk = shape
    p, seed, offset = 0.2, 1234, 9
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, dtype, seed=Sq + D)
    g = torch.Generator().manual_seed(Sk)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    dout = torch.randn(q.shape, generator=g).to(tdt)
    scale = softmax_scale(D)
    grads = run_bwd_dropout(q, k, v, dout, scale, causal, p, seed, offset)
    refs = oracle.attn_bwd_dropout(q, k, v, dout, scale, causal, dtype, p8_of(p), seed, offset, magnitudes=True)
    print(compare_bwd(grads, refs[:3], refs[3:], dtype, q, k, dout, scale, causal))


def test_backward_deterministic_and_p0():
    q, k, v = make_inputs(1, 2, 384, 128, "bf16", seed=1)
    g = torch.Generator().manual_seed(2)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    a = run_bwd_dropout(q, k, v, dout, 0.08, True, 0.3, 5, 6, deterministic=True)
    b = run_bwd_dropout(q, k, v, dout, 0.08, True, 0.3, 5, 6, deterministic=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    # p = 0: the same gradients as fa_bwd, bit for bit (deterministic mode)
    z = run_bwd_dropout(q, k, v, dout, 0.08, True, 0.0, 5, 6, deterministic=True)
    dq_, dk_, dv_, ddo = (t.cuda() for t in (q, k, v, dout))
    o, lse = fa.flash_attention_forward(dq_, dk_, dv_, 0.08, True)
    ref = fa.flash_attention_backward(dq_, dk_, dv_, o, lse, ddo, 0.08, True, deterministic=True)
    torch.cuda.synchronize()
    for x, y in zip(z, ref):
        assert torch.equal(x, y.cpu())


def test_full_size_sampled_rows():
    """The bench's long-context shape (1 x 32 x 16384 x 128, bf16, causal) with
    dropout 0.1: sampled rows against the oracle."""
    from tiled_attention_18_b200.workloads import sample_rows
    B, H, S, D = 1, 32, 16384, 128
    q, k, v = make_inputs(B, H, S, D, "bf16", seed=0)
    o, lse = run_fwd_dropout(q, k, v, softmax_scale(D), True, 0.1, seed=2024, offset=11)
    bh, rows = sample_rows(B, H, S, n_random=48, edge=2, seed=7)
    o_ref, lse_ref = oracle.attn_rows_dropout(q, k, v, softmax_scale(D), True, "bf16", p8_of(0.1), 2024, 11, bh, rows)
    og = o.view(B * H, S, D)[torch.as_tensor(bh), torch.as_tensor(rows)]
    lg = lse.view(B * H, S)[torch.as_tensor(bh), torch.as_tensor(rows)]
    check_o(og, lg, o_ref, lse_ref, "bf16", 0.1)

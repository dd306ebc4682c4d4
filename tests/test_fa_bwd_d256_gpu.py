"""GPU parity of the head-dimension-256 backward pass against the fp64 oracle.

A work unit of the D = 256 backward is (head, 128-key tile, half of D): both
halves recompute the full-D scores and form their own 128 columns of dK, dV
and dQ.  Each gradient element is compared with the oracle's exact gradient
within the suite's backward bound (gpu_helpers.compare_bwd); ragged and cross
shapes cover the partial key tiles and query steps, and the deterministic
mode must repeat bit for bit with its dQ turn counters kept per half.
"""
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import make_cross_inputs, softmax_scale

from gpu_helpers import compare_bwd, run_fa_bwd

pytestmark = pytest.mark.gpu

D = 256


def _dout(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.float16 if dtype == "fp16" else torch.bfloat16)


SHAPES = [(1, 1, 1, 1), (1, 2, 64, 64), (1, 1, 129, 129), (2, 1, 255, 255), (1, 2, 300, 300), (1, 1, 77, 300),
          (1, 2, 300, 77), (1, 1, 640, 700)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_d256_backward_matches_oracle(shape, dtype, causal):
    B, H, Sq, Sk = shape
    if causal and Sq > Sk:
        pytest.skip("causal needs Sq <= Sk")
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, dtype, seed=7 * Sq + Sk)
    dout = _dout(q.shape, dtype, seed=Sq + 3 * Sk)
    scale = softmax_scale(D)
    gq, gk, gv, _, _ = run_fa_bwd(q, k, v, dout, scale, causal)
    dq, dk, dv, mq, mk, mv = oracle.attn_bwd(q, k, v, dout, scale, causal, dtype, magnitudes=True)
    print(shape, dtype, causal, compare_bwd((gq, gk, gv), (dq, dk, dv), (mq, mk, mv), dtype, q, k, dout, scale,
                                            causal))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_d256_deterministic_repeats_bitwise(causal):
    q, k, v = make_cross_inputs(1, 3, 400, 520, D, "bf16", seed=5)
    dout = _dout(q.shape, "bf16", seed=6)
    scale = softmax_scale(D)
    runs = [run_fa_bwd(q, k, v, dout, scale, causal, deterministic=True)[:3] for _ in range(2)]
    for a, b in zip(*runs):
        assert torch.equal(a, b)
    dq, dk, dv, mq, mk, mv = oracle.attn_bwd(q, k, v, dout, scale, causal, "bf16", magnitudes=True)
    compare_bwd(runs[0], (dq, dk, dv), (mq, mk, mv), "bf16", q, k, dout, scale, causal)


def test_d256_strided_backward_equals_contiguous():
    """BSHD views through fa_bwd_ex give the contiguous call's gradients bit for bit."""
    B, H, S = 2, 2, 300
    q, k, v = make_cross_inputs(B, H, S, S, D, "bf16", seed=9)
    dout = _dout(q.shape, "bf16", seed=10)
    scale = softmax_scale(D)
    ref = run_fa_bwd(q, k, v, dout, scale, True)[:3]
    bshd = lambda t: t.transpose(1, 2).contiguous().cuda().transpose(1, 2)  # noqa: E731
    dq_, dk_, dv_, ddo = (bshd(t) for t in (q, k, v, dout))
    o, lse = fa.flash_attention_forward(dq_, dk_, dv_, scale, True)
    grads = fa.flash_attention_backward(dq_, dk_, dv_, o, lse, ddo, scale, True)
    assert fa.fa_check_status(torch.cuda.current_stream().cuda_stream) == 0
    for a, b in zip(grads, ref):
        assert torch.equal(a.contiguous().cpu(), b)


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_d256_masked_and_dropout_backward(causal):
    """The explicit mask and dropout paths of the D = 256 backward (fa_backward)."""
    B, H, Sq, Sk = 1, 2, 200, 260
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, "bf16", seed=13)
    dout = _dout(q.shape, "bf16", seed=14)
    scale = softmax_scale(D)
    g = torch.Generator().manual_seed(15)
    mask = torch.rand((1, H, Sq, Sk), generator=g) < 0.7
    i = torch.arange(Sq)
    mask[..., i, torch.clamp(i + (Sk - Sq), max=Sk - 1)] = True
    dq_, dk_, dv_, ddo = (t.cuda() for t in (q, k, v, dout))
    pad = -(-Sk // 16) * 16
    mbuf = torch.zeros((1, H, Sq, pad), dtype=torch.uint8)
    mbuf[..., :Sk] = mask.to(torch.uint8)
    dm = mbuf.cuda()[..., :Sk]
    o, lse = fa.flash_attention_forward(dq_, dk_, dv_, scale, causal, mask=dm)
    grads = fa.flash_attention_backward(dq_, dk_, dv_, o, lse, ddo, scale, causal, mask=dm)
    assert fa.fa_check_status(torch.cuda.current_stream().cuda_stream) == 0
    refs = oracle.attn_bwd_masked(q, k, v, dout, mask, scale, causal, "bf16", magnitudes=True)
    compare_bwd(tuple(t.cpu() for t in grads), refs[:3], refs[3:], "bf16", q, k, dout, scale, causal)

    p, seed, offset = 0.2, 4321, 3
    o, lse = fa.flash_attention_forward(dq_, dk_, dv_, scale, causal, dropout_p=p, seed=seed, offset=offset)
    grads = fa.flash_attention_backward(dq_, dk_, dv_, o, lse, ddo, scale, causal, dropout_p=p, seed=seed,
                                        offset=offset)
    assert fa.fa_check_status(torch.cuda.current_stream().cuda_stream) == 0
    p8 = int(p * 256 + 0.5)
    refs = oracle.attn_bwd_dropout(q, k, v, dout, scale, causal, "bf16", p8, seed, offset, magnitudes=True)
    compare_bwd(tuple(t.cpu() for t in grads), refs[:3], refs[3:], "bf16", q, k, dout, scale, causal)

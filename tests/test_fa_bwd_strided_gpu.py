"""fa_bwd_ex: the backward pass on strided tensors (BSHD views, packed QKV,
padded gradient buffers) against the fp64 oracle, and bit for bit against
fa_bwd on contiguous copies of the same data (deterministic dQ order)."""
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import make_cross_inputs, softmax_scale

from gpu_helpers import compare_bwd

pytestmark = pytest.mark.gpu


def bshd_view(x):
    """The same values as BHSD x, stored as [B, S, H, D] and viewed as BHSD."""
    return x.transpose(1, 2).contiguous().transpose(1, 2)


def run(q, k, v, dout, scale, causal, layout, deterministic=True):
    """Forward + backward on the GPU with the inputs (and O, dO, gradients) in
    the given layout; returns contiguous CPU gradients."""
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    dq_, dk_, dv_, ddo = (t.cuda() for t in (q, k, v, dout))
    if layout == "bshd":
        dq_, dk_, dv_, ddo = (bshd_view(t) for t in (dq_, dk_, dv_, ddo))
        o = bshd_view(torch.empty_like(dq_))
        gq, gk, gv = (bshd_view(torch.empty_like(t)) for t in (dq_, dk_, dv_))
    elif layout == "packed":
        # Q, K, V interleaved per position ([B, S, 3, H, D]; needs Sq = Sk); gradients in
        # buffers whose rows are padded by 16 elements
        qkv = torch.stack([t.transpose(1, 2) for t in (dq_, dk_, dv_)], dim=2).contiguous()
        dq_, dk_, dv_ = (qkv[:, :, i].transpose(1, 2) for i in range(3))
        o = torch.empty_like(dq_.contiguous())
        pad = lambda t: torch.empty(B, H, t.shape[2], D + 16, dtype=t.dtype, device="cuda")[..., :D]  # noqa: E731
        gq, gk, gv = pad(dq_), pad(dk_), pad(dv_)
    else:
        o = torch.empty_like(dq_)
        gq, gk, gv = (torch.empty_like(t) for t in (dq_, dk_, dv_))
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device="cuda")
    fa.flash_attention_forward(dq_, dk_, dv_, scale, causal, out=o, lse=lse)
    fa.flash_attention_backward(dq_, dk_, dv_, o, lse, ddo, scale, causal, deterministic=deterministic,
                                dq=gq, dk=gk, dv=gv)
    st = fa.fa_check_status(torch.cuda.current_stream().cuda_stream)
    assert st == 0, fa.fa_status_string(st)
    return tuple(t.contiguous().cpu() for t in (gq, gk, gv))


@pytest.mark.parametrize("layout", ["bshd", "packed"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("fp16", 64)])
def test_strided_backward_matches_oracle_and_contiguous(layout, causal, dtype, D):
    B, H, S = 2, 3, 257
    q, k, v = make_cross_inputs(B, H, S, S, D, dtype, seed=D + causal)
    g = torch.Generator().manual_seed(3)
    dout = torch.randn(q.shape, generator=g).to(q.dtype)
    scale = softmax_scale(D)
    grads = run(q, k, v, dout, scale, causal, layout)
    refs = oracle.attn_bwd(q, k, v, dout, scale, causal, dtype, magnitudes=True)
    print(compare_bwd(grads, refs[:3], refs[3:], dtype, q, k, dout, scale, causal))
    same = run(q, k, v, dout, scale, causal, "bhsd")
    for a, b in zip(grads, same):
        assert torch.equal(a, b)


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_strided_backward_cross_shapes(causal):
    q, k, v = make_cross_inputs(1, 4, 190, 300, 128, "bf16", seed=11)
    g = torch.Generator().manual_seed(12)
    dout = torch.randn(q.shape, generator=g).to(q.dtype)
    grads = run(q, k, v, dout, 0.09, causal, "bshd", deterministic=False)
    refs = oracle.attn_bwd(q, k, v, dout, 0.09, causal, "bf16", magnitudes=True)
    compare_bwd(grads, refs[:3], refs[3:], "bf16", q, k, dout, 0.09, causal)

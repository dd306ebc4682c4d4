"""The autograd wiring of ``tiled_attention_18_b200.autograd.attention`` on
CPU: the two kernel calls are replaced by float64 stand-ins (the oracle's
forward and a direct gradient formula), so the test checks what the module
adds -- saved tensors, argument passing, the gradient routing -- against
torch autograd of the same attention."""
import numpy as np
import pytest
import torch

import oracle
from tiled_attention_18_b200 import autograd as fa_autograd
from tiled_attention_18_b200.workloads import make_cross_inputs


def _fake_forward(q, k, v, scale, causal, dropout_p=0.0, seed=0, offset=0, mask=None):
    assert dropout_p == 0.0 and mask is None
    o, lse = oracle.attn_fwd_gen(q.detach(), k.detach(), v.detach(), scale, causal, "bf16")
    return torch.from_numpy(o), torch.from_numpy(lse)


def _fake_backward(q, k, v, o, lse, do, scale, causal, deterministic=False, dropout_p=0.0, seed=0, offset=0,
                   mask=None):
    assert do.is_contiguous()
    qd, kd, vd, dod = (t.detach().double() for t in (q, k, v, do))
    s = scale * qd @ kd.transpose(-1, -2)
    if causal:
        Sq, Sk = s.shape[-2:]
        s = s.masked_fill(torch.arange(Sk)[None, :] > torch.arange(Sq)[:, None] + (Sk - Sq), float("-inf"))
    p = torch.exp(s - lse[..., None])
    ds = p * (dod @ vd.transpose(-1, -2) - (dod * o).sum(-1, keepdim=True))
    return scale * ds @ kd, scale * ds.transpose(-1, -2) @ qd, p.transpose(-1, -2) @ dod


@pytest.mark.parametrize("causal", [False, True])
def test_attention_function_routes_gradients(monkeypatch, causal):
    monkeypatch.setattr(fa_autograd, "_forward", _fake_forward)
    monkeypatch.setattr(fa_autograd, "_backward", _fake_backward)
    q, k, v = make_cross_inputs(1, 2, 20, 30, 8, "bf16", seed=1)
    tq, tk, tv = (t.double().requires_grad_(True) for t in (q, k, v))
    # the function receives the 16-bit tensors (what the kernels take); gradients come back in float64
    q16, k16, v16 = (t.clone().requires_grad_(True) for t in (q, k, v))
    o, lse = fa_autograd.attention(q16, k16, v16, scale=0.375, causal=causal, return_lse=True)
    assert not lse.requires_grad
    dout = torch.randn(o.shape, generator=torch.Generator().manual_seed(2), dtype=torch.float64)
    # a non-contiguous upstream gradient: the module must hand the kernel a dense one
    (o * dout.transpose(-1, -2).contiguous().transpose(-1, -2)).sum().backward()
    s = 0.375 * tq @ tk.transpose(-1, -2)
    if causal:
        s = s.masked_fill(torch.arange(30)[None, :] > torch.arange(20)[:, None] + 10, float("-inf"))
    (torch.softmax(s, -1) @ tv * dout).sum().backward()
    # autograd hands back each gradient in its input's dtype (bf16): one rounding
    for mine, ref in ((q16.grad, tq.grad), (k16.grad, tk.grad), (v16.grad, tv.grad)):
        assert mine.dtype == torch.bfloat16
        assert np.allclose(mine.double().numpy(), ref.numpy(), rtol=2.0 ** -8, atol=1e-6)


def test_default_scale_is_inverse_sqrt_d(monkeypatch):
    seen = {}

    def fake(q, k, v, scale, causal, **kw):
        seen["scale"] = scale
        return _fake_forward(q, k, v, scale, causal, **kw)

    monkeypatch.setattr(fa_autograd, "_forward", fake)
    q, k, v = make_cross_inputs(1, 1, 4, 4, 16, "bf16", seed=3)
    fa_autograd.attention(q, k, v)
    assert seen["scale"] == 16 ** -0.5

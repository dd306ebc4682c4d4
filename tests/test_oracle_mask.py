"""Pins for the explicit-mask oracle (CPU only)."""
import numpy as np
import pytest
import torch

import oracle
from tiled_attention_18_b200.workloads import make_cross_inputs, make_inputs, softmax_scale


def _random_mask(shape, seed, p_keep=0.7):
    g = torch.Generator().manual_seed(seed)
    return torch.rand(shape, generator=g) < p_keep


@pytest.mark.parametrize("mshape", ["full", "bcast_b", "bcast_h", "bcast_both"])
@pytest.mark.parametrize("causal", [False, True])
def test_masked_matches_sdpa_fp64(mshape, causal):
    B, H, Sq, Sk, D = 2, 3, 33, 50, 16
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, "bf16", seed=7)
    shape = {"full": (B, H, Sq, Sk), "bcast_b": (1, H, Sq, Sk), "bcast_h": (B, 1, Sq, Sk),
             "bcast_both": (1, 1, Sq, Sk)}[mshape]
    mask = _random_mask(shape, seed=3)
    mask[..., 0] = True                      # every row keeps key 0 (no empty rows here)
    scale = softmax_scale(D)
    o, lse = oracle.attn_fwd_masked(q, k, v, mask, scale, causal, "bf16")
    full = mask.expand(B, H, Sq, Sk)
    if causal:
        i = torch.arange(Sq)[:, None]
        j = torch.arange(Sk)[None, :]
        full = full & (j <= i + (Sk - Sq))
    q64, k64, v64 = (t.to(torch.float64) for t in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(q64, k64, v64, attn_mask=full, scale=float(scale))
    assert np.max(np.abs(o - ref.numpy())) <= 1e-12
    s = (q64 @ k64.transpose(-1, -2)) * float(scale)
    ref_lse = torch.logsumexp(s.masked_fill(~full, float("-inf")), dim=-1)
    assert np.max(np.abs(lse - ref_lse.numpy())) <= 1e-12


def test_all_ones_mask_equals_no_mask_and_tril_equals_causal():
    q, k, v = make_inputs(1, 2, 40, 16, "fp16", seed=5)
    ones = torch.ones(1, 1, 40, 40, dtype=torch.bool)
    for causal in (False, True):
        a = oracle.attn_fwd_gen(q, k, v, 0.3, causal, "fp16")
        b = oracle.attn_fwd_masked(q, k, v, ones, 0.3, causal, "fp16")
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    tril = torch.tril(torch.ones(40, 40, dtype=torch.bool))[None, None]
    a = oracle.attn_fwd_gen(q, k, v, 0.3, True, "fp16")
    b = oracle.attn_fwd_masked(q, k, v, tril, 0.3, False, "fp16")
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_fully_masked_rows_are_zero_with_minus_infinite_lse():
    q, k, v = make_cross_inputs(1, 2, 10, 20, 8, "bf16", seed=1)
    mask = _random_mask((1, 2, 10, 20), seed=2)
    mask[0, 0, 3] = False
    mask[0, 1, 7] = False
    o, lse = oracle.attn_fwd_masked(q, k, v, mask, 0.5, False, "bf16")
    assert np.all(o[0, 0, 3] == 0) and np.isneginf(lse[0, 0, 3])
    assert np.all(o[0, 1, 7] == 0) and np.isneginf(lse[0, 1, 7])
    assert np.isfinite(lse[0, 0, 2])


def test_single_kept_key_gives_its_value():
    q, k, v = make_cross_inputs(1, 1, 6, 9, 8, "fp16", seed=4)
    mask = torch.zeros(1, 1, 6, 9, dtype=torch.bool)
    for i in range(6):
        mask[0, 0, i, (2 * i + 1) % 9] = True
    o, _ = oracle.attn_fwd_masked(q, k, v, mask, 0.5, False, "fp16")
    for i in range(6):
        assert np.array_equal(o[0, 0, i], v[0, 0, (2 * i + 1) % 9].to(torch.float64).numpy())


def _dout(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("causal", [False, True])
def test_masked_bwd_matches_fp64_autograd(causal):
    B, H, Sq, Sk, D = 2, 2, 20, 30, 8
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, "bf16", seed=13)
    mask = _random_mask((1, H, Sq, Sk), seed=14)
    mask[..., 0] = True
    dout = _dout(q.shape, 15)
    dq, dk, dv = oracle.attn_bwd_masked(q, k, v, dout, mask, 0.4, causal, "bf16")
    full = mask.expand(B, H, Sq, Sk)
    if causal:
        full = full & (torch.arange(Sk)[None, :] <= torch.arange(Sq)[:, None] + (Sk - Sq))
    q64, k64, v64 = (t.to(torch.float64).requires_grad_(True) for t in (q, k, v))
    s = (q64 @ k64.transpose(-1, -2)) * float(np.float32(0.4))
    o = torch.softmax(s.masked_fill(~full, float("-inf")), dim=-1) @ v64
    o.backward(dout.to(torch.float64))
    for a, b in ((dq, q64.grad), (dk, k64.grad), (dv, v64.grad)):
        assert np.max(np.abs(a - b.numpy())) <= 1e-12


def test_masked_bwd_all_ones_equals_unmasked_and_empty_rows_get_nothing():
    q, k, v = make_inputs(1, 2, 24, 8, "fp16", seed=16)
    dout = _dout(q.shape, 17).to(torch.float16)
    ones = torch.ones(1, 1, 24, 24, dtype=torch.bool)
    a = oracle.attn_bwd(q, k, v, dout, 0.3, True, "fp16")
    b = oracle.attn_bwd_masked(q, k, v, dout, ones, 0.3, True, "fp16")
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    mask = _random_mask((1, 2, 24, 24), seed=18)
    mask[..., 0] = True
    mask[0, 1, 5] = False        # row 5 of head 1 sees nothing
    dq, dk, dv = oracle.attn_bwd_masked(q, k, v, dout, mask, 0.3, False, "fp16")
    assert np.all(dq[0, 1, 5] == 0)
    # the empty row contributes nothing: the same gradients with its dO zeroed
    dout0 = dout.clone()
    dout0[0, 1, 5] = 0
    dq0, dk0, dv0 = oracle.attn_bwd_masked(q, k, v, dout0, mask, 0.3, False, "fp16")
    assert np.array_equal(dk, dk0) and np.array_equal(dv, dv0)

"""Pins for the general-shape oracle (Sq != Sk, causal aligned to the last Sq
keys).  CPU only."""
import numpy as np
import pytest
import torch

import oracle
from tiled_attention_18_b200.workloads import make_cross_inputs as _qkv
from tiled_attention_18_b200.workloads import make_inputs, softmax_scale


def _bottom_right_mask(Sq, Sk):
    i = torch.arange(Sq)[:, None]
    j = torch.arange(Sk)[None, :]
    return j <= i + (Sk - Sq)


@pytest.mark.parametrize("Sq,Sk", [(1, 1), (1, 37), (7, 33), (77, 130), (64, 64), (130, 64)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_general_oracle_matches_sdpa_fp64(Sq, Sk, causal, dtype):
    if causal and Sq > Sk:
        pytest.skip("rows with no visible key are checked separately")
    q, k, v = _qkv(2, 2, Sq, Sk, 16, dtype, seed=Sq * 31 + Sk)
    scale = softmax_scale(16)
    o, lse = oracle.attn_fwd_gen(q, k, v, scale, causal, dtype)
    mask = _bottom_right_mask(Sq, Sk) if causal else None
    q64, k64, v64 = (t.to(torch.float64) for t in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(q64, k64, v64, attn_mask=mask, scale=float(scale))
    assert np.max(np.abs(o - ref.numpy())) <= 1e-12
    s = torch.matmul(q64, k64.transpose(-1, -2)) * float(scale)
    if causal:
        s = s.masked_fill(~mask, float("-inf"))
    assert np.max(np.abs(lse - torch.logsumexp(s, dim=-1).numpy())) <= 1e-12


def test_general_equals_square_oracle_when_sq_equals_sk():
    q, k, v = make_inputs(1, 3, 45, 32, "bf16", seed=4)
    for causal in (False, True):
        a = oracle.attn_fwd(q, k, v, 0.2, causal, "bf16")
        b = oracle.attn_fwd_gen(q, k, v, 0.2, causal, "bf16")
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("causal", [False, True])
def test_general_zero_query_closed_form(causal):
    Sq, Sk = 20, 50
    _, k, v = _qkv(1, 2, Sq, Sk, 8, "fp16", seed=9)
    q = torch.zeros((1, 2, Sq, 8), dtype=torch.float16)
    o, lse = oracle.attn_fwd_gen(q, k, v, 0.3, causal, "fp16")
    vd = v.to(torch.float64).numpy()
    for i in range(Sq):
        n = i + (Sk - Sq) + 1 if causal else Sk
        assert np.max(np.abs(o[:, :, i] - vd[:, :, :n].mean(axis=2))) <= 1e-14
        assert np.max(np.abs(lse[:, :, i] - np.log(n))) <= 1e-14


def test_rows_without_keys_are_zero_with_minus_infinite_lse():
    q, k, v = _qkv(1, 1, 10, 4, 8, "bf16", seed=2)   # Sk - Sq = -6: rows 0..5 see nothing
    o, lse = oracle.attn_fwd_gen(q, k, v, 0.5, True, "bf16")
    assert np.all(o[0, 0, :6] == 0) and np.all(np.isneginf(lse[0, 0, :6]))
    assert np.all(np.isfinite(lse[0, 0, 6:]))


def test_general_rows_equal_full_run():
    q, k, v = _qkv(2, 2, 33, 90, 16, "fp16", seed=13)
    for causal in (False, True):
        o, lse = oracle.attn_fwd_gen(q, k, v, 0.25, causal, "fp16")
        bh = np.array([0, 0, 1, 3, 3, 2], dtype=np.int64)
        rows = np.array([0, 5, 32, 1, 17, 20], dtype=np.int64)
        orow, lrow = oracle.attn_rows_gen(q, k, v, 0.25, causal, "fp16", bh, rows)
        assert np.array_equal(orow, o.reshape(4, 33, 16)[bh, rows])
        assert np.array_equal(lrow, lse.reshape(4, 33)[bh, rows])

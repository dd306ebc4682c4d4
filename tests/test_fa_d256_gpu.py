"""GPU parity of the head-dimension-256 forward kernel (fa_fwd / fa_fwd_ex with
D = 256, through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from tiled_attention_18_b200.workloads import make_cross_inputs, make_inputs, sample_rows, softmax_scale

from gpu_helpers import compare, run_fa, run_fa_ex

pytestmark = pytest.mark.gpu

SHAPES = [
    # (B, H, Sq, Sk)
    (1, 1, 1, 1), (1, 2, 17, 17), (1, 1, 64, 64), (1, 2, 128, 128), (2, 1, 129, 129), (1, 2, 255, 300),
    (1, 1, 300, 77), (2, 2, 513, 513), (1, 3, 100, 1000),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_d256_matches_oracle(shape, dtype, causal):
    B, H, Sq, Sk = shape
    if causal and Sq > Sk:
        pytest.skip("causal needs Sq <= Sk")
    q, k, v = make_cross_inputs(B, H, Sq, Sk, 256, dtype, seed=Sq + 7 * Sk)
    scale = softmax_scale(256)
    if Sq == Sk:
        o, lse = run_fa(q, k, v, scale, causal)
    else:
        o, lse = run_fa_ex(q, k, v, scale, causal)
    o_ref, lse_ref = oracle.attn_fwd_gen(q, k, v, scale, causal, dtype)
    print(shape, dtype, causal, compare(o, lse, o_ref, lse_ref, dtype))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_d256_strided_layouts_bitwise_equal_contiguous(causal):
    q, k, v = make_cross_inputs(2, 3, 200, 333, 256, "bf16", seed=3)
    a = run_fa_ex(q, k, v, 0.0625, causal, layouts=("bshd",) * 4)
    b = run_fa_ex(q, k, v, 0.0625, causal)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    o_ref, lse_ref = oracle.attn_fwd_gen(q, k, v, 0.0625, causal, "bf16")
    compare(a[0], a[1], o_ref, lse_ref, "bf16")


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_d256_zero_query_closed_form(causal):
    B, H, S = 1, 2, 1000
    _, k, v = make_inputs(B, H, S, 256, "bf16", seed=4)
    q = torch.zeros_like(k)
    o, lse = run_fa(q, k, v, 0.0625, causal)
    vd = v.to(torch.float64).numpy()
    n = np.arange(1, S + 1, dtype=np.float64)
    if causal:
        ref = np.cumsum(vd, axis=2) / n[None, None, :, None]
        ref_lse = np.broadcast_to(np.log(n), (B, H, S))
    else:
        ref = np.broadcast_to(vd.mean(axis=2, keepdims=True), vd.shape)
        ref_lse = np.full((B, H, S), np.log(S))
    compare(o, lse, ref, ref_lse, "bf16")


def test_d256_long_causal_sampled_rows():
    B, H, S = 1, 8, 8192
    q, k, v = make_inputs(B, H, S, 256, "bf16", seed=5)
    scale = softmax_scale(256)
    o, lse = run_fa(q, k, v, scale, True)
    bh, rows = sample_rows(B, H, S, n_random=512, edge=2)
    o_ref, lse_ref = oracle.attn_rows(q, k, v, scale, True, "bf16", bh, rows)
    og = o.reshape(B * H, S, 256)[torch.from_numpy(bh), torch.from_numpy(rows)]
    lg = lse.reshape(B * H, S)[torch.from_numpy(bh), torch.from_numpy(rows)]
    print(compare(og, lg, o_ref, lse_ref, "bf16"))
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    assert torch.equal(o[:, :, 0], v[:, :, 0])

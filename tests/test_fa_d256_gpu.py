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


def _p8(p):
    return int(np.floor(p * 256 + 0.5))


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("shape", [(2, 2, 200, 200), (1, 3, 130, 333)], ids=["square", "cross"])
def test_d256_explicit_mask(dtype, causal, shape):
    """D = 256 with an explicit per-head mask (some rows fully masked)."""
    import tiled_attention_18_b200 as fa
    B, H, Sq, Sk = shape
    q, k, v = make_cross_inputs(B, H, Sq, Sk, 256, dtype, seed=Sk)
    pad = (Sk + 15) // 16 * 16
    g = torch.Generator().manual_seed(Sq)
    m = (torch.rand(B, H, Sq, pad, generator=g) < 0.7).to(torch.uint8)
    m[:, :, 3] = 0  # an empty row: O = 0, LSE = -inf
    scale = softmax_scale(256)
    o, lse = fa.flash_attention_forward(q.cuda(), k.cuda(), v.cuda(), scale, causal, mask=m.cuda()[..., :Sk])
    assert fa.fa_check_status(torch.cuda.current_stream().cuda_stream) == 0
    o_ref, lse_ref = oracle.attn_fwd_masked(q, k, v, m[..., :Sk].numpy(), scale, causal, dtype)
    og, lg = o.cpu(), lse.cpu().double().numpy()
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lg), empty)
    lg[empty] = 0.0
    lse_ref = np.where(empty, 0.0, lse_ref)
    compare(og, torch.from_numpy(lg), o_ref, lse_ref, dtype)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_d256_dropout_keep_decisions_and_values(dtype):
    """V = identity over 256 keys gives the keep decisions bit for bit; then the
    values of a causal cross-shaped call against the oracle."""
    import tiled_attention_18_b200 as fa
    from gpu_helpers import half_ulp
    from tiled_attention_18_b200.workloads import LSE_TOL, O_TOL
    B, H, S, D, p = 1, 2, 256, 256, 0.2
    q, k, _ = make_inputs(B, H, S, D, dtype, seed=1)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    eye = torch.eye(D, dtype=tdt).expand(B, H, D, D).contiguous()
    o, _ = fa.flash_attention_forward(q.cuda(), k.cuda(), eye.cuda(), softmax_scale(D), False, dropout_p=p, seed=5,
                                      offset=6)
    torch.cuda.synchronize()
    keep = oracle.dropout_keep_mask(B * H, S, S, _p8(p), 5, 6).reshape(B, H, S, S)
    assert np.array_equal(o.cpu().float().numpy() != 0, keep.astype(bool))
    q, k, v = make_cross_inputs(2, 2, 150, 260, D, dtype, seed=2)
    o, lse = fa.flash_attention_forward(q.cuda(), k.cuda(), v.cuda(), softmax_scale(D), True, dropout_p=p, seed=7,
                                        offset=8)
    o_ref, lse_ref = oracle.attn_fwd_dropout(q, k, v, softmax_scale(D), True, dtype, _p8(p), 7, 8)
    zs = 256.0 / (256.0 - _p8(p))
    err = np.abs(o.cpu().double().numpy() - o_ref)
    rep = half_ulp(o_ref, dtype) < O_TOL[dtype] * zs
    assert err[rep].max() <= O_TOL[dtype] * zs
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= LSE_TOL


def test_d256_mask_and_dropout_on_bshd_views():
    import tiled_attention_18_b200 as fa
    from gpu_helpers import half_ulp
    from tiled_attention_18_b200.workloads import O_TOL
    B, H, Sq, Sk, D, p = 2, 2, 140, 200, 256, 0.1
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, "bf16", seed=4)
    bshd = lambda t: t.cuda().transpose(1, 2).contiguous().transpose(1, 2)  # noqa: E731
    m = torch.zeros(B, 1, Sq, 208, dtype=torch.uint8)
    m[0, :, :, :150] = 1
    m[1, :, :, :200] = 1
    o = bshd(torch.empty(q.shape, dtype=q.dtype))
    o, lse = fa.flash_attention_forward(bshd(q), bshd(k), bshd(v), 0.0625, False, out=o, dropout_p=p, seed=9,
                                        offset=10, mask=m.cuda()[..., :Sk])
    torch.cuda.synchronize()
    o_ref, _ = oracle.attn_fwd_dropout(q, k, v, 0.0625, False, "bf16", _p8(p), 9, 10, mask=m[..., :Sk].numpy())
    zs = 256.0 / (256.0 - _p8(p))
    err = np.abs(o.contiguous().cpu().double().numpy() - o_ref)
    rep = half_ulp(o_ref, "bf16") < O_TOL["bf16"] * zs
    assert err[rep].max() <= O_TOL["bf16"] * zs

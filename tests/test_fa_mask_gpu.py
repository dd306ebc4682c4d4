"""GPU parity of fa_fwd_mask (explicit boolean mask fused into the forward
kernel, through the C ABI) against the fp64 masked oracle."""
import numpy as np
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import make_cross_inputs, make_inputs, softmax_scale

from gpu_helpers import compare, run_fa_ex

pytestmark = pytest.mark.gpu


def _device_mask(mask_bool: torch.Tensor):
    """uint8 device copy with rows padded to a multiple of 16 bytes; returns
    (tensor, (b, h, row) element strides with 0 over broadcast dimensions)."""
    Bm, Hm, Sq, Sk = mask_bool.shape
    pad = -(-Sk // 16) * 16
    buf = torch.zeros((Bm, Hm, Sq, pad), dtype=torch.uint8)
    buf[..., :Sk] = mask_bool.to(torch.uint8)
    d = buf.cuda()
    sb = 0 if Bm == 1 else Hm * Sq * pad
    sh = 0 if Hm == 1 else Sq * pad
    return d, (sb, sh, pad)


def run_masked(q, k, v, mask_bool, scale, causal):
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    o = torch.full_like(dq, float("nan"))
    lse = torch.full((B, H, Sq), float("nan"), dtype=torch.float32, device="cuda")
    dm, ms = _device_mask(mask_bool)
    st = torch.cuda.current_stream().cuda_stream
    dt = fa.FA_BF16 if q.dtype == torch.bfloat16 else fa.FA_FP16
    rc = fa.fa_fwd_mask(dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, Sq, Sk, D,
                        dm.data_ptr(), ms, scale, int(causal), dt, st)
    assert rc == 0, f"fa_fwd_mask returned {rc} ({fa.fa_status_string(rc)})"
    s = fa.fa_check_status(st)
    assert s == 0, f"device status {s}"
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def _mask(shape, seed, p_keep=0.6):
    g = torch.Generator().manual_seed(seed)
    m = torch.rand(shape, generator=g) < p_keep
    m[..., 0] = True          # no empty rows (checked separately)
    return m


CASES = [
    # (B, H, Sq, Sk, D, mask dims)
    (1, 2, 200, 200, 64, "full"), (2, 3, 129, 300, 128, "bcast_b"), (1, 4, 300, 333, 64, "bcast_h"),
    (2, 2, 256, 700, 128, "bcast_both"), (1, 1, 77, 1000, 128, "full"), (1, 2, 513, 513, 64, "bcast_both"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_masked_matches_oracle(case, dtype, causal):
    B, H, Sq, Sk, D, md = case
    if causal and Sq > Sk:
        pytest.skip("causal needs Sq <= Sk")
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, dtype, seed=Sq + Sk)
    shape = {"full": (B, H, Sq, Sk), "bcast_b": (1, H, Sq, Sk), "bcast_h": (B, 1, Sq, Sk),
             "bcast_both": (1, 1, Sq, Sk)}[md]
    mask = _mask(shape, seed=Sq * 3 + Sk)
    if causal:
        # keep each row's last visible key too, so that no row is empty under both masks
        i = torch.arange(Sq)
        mask[..., i, torch.clamp(i + (Sk - Sq), max=Sk - 1)] = True
    scale = softmax_scale(D)
    o, lse = run_masked(q, k, v, mask, scale, causal)
    o_ref, lse_ref = oracle.attn_fwd_masked(q, k, v, mask, scale, causal, dtype)
    print(compare(o, lse, o_ref, lse_ref, dtype))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_all_ones_mask_equals_unmasked_bitwise(causal):
    q, k, v = make_cross_inputs(2, 3, 300, 500, 128, "bf16", seed=8)
    ones = torch.ones(1, 1, 300, 500, dtype=torch.bool)
    a = run_masked(q, k, v, ones, 0.1, causal)
    b = run_fa_ex(q, k, v, 0.1, causal)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_tril_mask_equals_causal_flag_bitwise(dtype):
    q, k, v = make_inputs(1, 4, 777, 64, dtype, seed=9)
    tril = torch.tril(torch.ones(777, 777, dtype=torch.bool))[None, None]
    a = run_masked(q, k, v, tril, 0.125, False)
    b = run_fa_ex(q, k, v, 0.125, True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_fully_masked_rows_give_zero_and_minus_infinity():
    q, k, v = make_cross_inputs(1, 2, 300, 400, 64, "fp16", seed=10)
    mask = _mask((1, 2, 300, 400), seed=11)
    empty = [3, 128, 129, 255, 299]
    mask[0, 0, empty] = False
    mask[0, 1, 17] = False
    o, lse = run_masked(q, k, v, mask, 0.125, False)
    o_ref, lse_ref = oracle.attn_fwd_masked(q, k, v, mask, 0.125, False, "fp16")
    for h, rows in ((0, empty), (1, [17])):
        assert torch.all(o[0, h, rows] == 0)
        assert torch.all(torch.isneginf(lse[0, h, rows]))
    keep = np.isfinite(lse_ref)
    og, lg = o.numpy(), lse.numpy()
    assert np.max(np.abs(og[keep] - o_ref[keep])) <= 2e-3
    assert np.max(np.abs(lg[keep] - lse_ref[keep])) <= 1e-3


def test_block_sparse_mask_long_sequence():
    """S = 4096, D = 128, bf16, a block-sparse mask (local windows plus a few
    global keys) shared by all heads: every output row against the oracle."""
    B, H, S, D = 1, 2, 4096, 128
    q, k, v = make_inputs(B, H, S, D, "bf16", seed=12)
    i = torch.arange(S)[:, None]
    j = torch.arange(S)[None, :]
    mask = ((i // 256) == (j // 256)) | (j < 64) | ((j % 512) == 7)
    mask = mask[None, None]
    o, lse = run_masked(q, k, v, mask, softmax_scale(D), False)
    o_ref, lse_ref = oracle.attn_fwd_masked(q, k, v, mask, softmax_scale(D), False, "bf16")
    print(compare(o, lse, o_ref, lse_ref, "bf16"))


def _dout(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.float16 if dtype == "fp16" else torch.bfloat16)


def run_masked_bwd(q, k, v, dout, mask_bool, scale, causal, deterministic=False):
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    dq_, dk_, dv_, ddo = (t.cuda() for t in (q, k, v, dout))
    o = torch.empty_like(dq_)
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device="cuda")
    dm, ms = _device_mask(mask_bool)
    st = torch.cuda.current_stream().cuda_stream
    dt = fa.FA_BF16 if q.dtype == torch.bfloat16 else fa.FA_FP16
    assert fa.fa_fwd_mask(dq_.data_ptr(), dk_.data_ptr(), dv_.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, Sq, Sk,
                          D, dm.data_ptr(), ms, scale, int(causal), dt, st) == 0
    gq, gk, gv = (torch.full_like(t, float("nan")) for t in (dq_, dk_, dv_))
    nb = fa.fa_bwd_workspace_size(B, H, Sq, D)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    rc = fa.fa_bwd_mask(dq_.data_ptr(), dk_.data_ptr(), dv_.data_ptr(), o.data_ptr(), ddo.data_ptr(), lse.data_ptr(),
                        gq.data_ptr(), gk.data_ptr(), gv.data_ptr(), ws.data_ptr(), nb, B, H, Sq, Sk, D,
                        dm.data_ptr(), ms, scale, int(causal), int(deterministic), dt, st)
    assert rc == 0, f"fa_bwd_mask returned {rc}"
    assert fa.fa_check_status(st) == 0
    torch.cuda.synchronize()
    return gq.cpu(), gk.cpu(), gv.cpu()


BWD_CASES = [(1, 2, 200, 200, 64, "full"), (2, 2, 129, 300, 128, "bcast_b"), (1, 3, 300, 333, 64, "bcast_both"),
             (1, 2, 256, 700, 128, "full")]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "x".join(map(str, c)))
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_masked_bwd_matches_oracle(case, dtype, causal):
    from gpu_helpers import compare_bwd
    B, H, Sq, Sk, D, md = case
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, dtype, seed=Sq + 2 * Sk)
    shape = {"full": (B, H, Sq, Sk), "bcast_b": (1, H, Sq, Sk), "bcast_both": (1, 1, Sq, Sk)}[md]
    mask = _mask(shape, seed=Sq + Sk)
    if causal:
        i = torch.arange(Sq)
        mask[..., i, torch.clamp(i + (Sk - Sq), max=Sk - 1)] = True
    mask[..., 5, :] = False                      # a row that sees no key
    dout = _dout(q.shape, dtype, seed=Sq)
    scale = softmax_scale(D)
    gq, gk, gv = run_masked_bwd(q, k, v, dout, mask, scale, causal)
    dq, dk, dv, mq, mk, mv = oracle.attn_bwd_masked(q, k, v, dout, mask, scale, causal, dtype, magnitudes=True)
    # the subnormal term's absolute sums run over every causally visible pair, masked
    # ones included: a looser, still valid bound
    print(compare_bwd((gq, gk, gv), (dq, dk, dv), (mq, mk, mv), dtype, q, k, dout, scale, causal))
    assert torch.all(gq[:, :, 5] == 0)


def test_masked_bwd_deterministic_repeatable():
    q, k, v = make_inputs(1, 4, 2048, 128, "bf16", seed=31)
    dout = _dout(q.shape, "bf16", seed=32)
    i = torch.arange(2048)[:, None]
    j = torch.arange(2048)[None, :]
    mask = (((i // 128) == (j // 128)) | (j < 32))[None, None]
    a = run_masked_bwd(q, k, v, dout, mask, 0.088, False, deterministic=True)
    b = run_masked_bwd(q, k, v, dout, mask, 0.088, False, deterministic=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    from gpu_helpers import compare_bwd
    dq, dk, dv, mq, mk, mv = oracle.attn_bwd_masked(q, k, v, dout, mask, 0.088, False, "bf16", magnitudes=True)
    print(compare_bwd(a, (dq, dk, dv), (mq, mk, mv), "bf16", q, k, dout, 0.088, False))

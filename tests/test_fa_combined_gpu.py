"""fa_forward / fa_backward: options combined in one call -- BSHD views, a
key-padding mask, dropout, Sq != Sk and the causal mask -- against the fp64
oracle; the combined keep/mask decisions bit-exact (V = identity); without
options, bit for bit the plain entries."""
import numpy as np
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import LSE_TOL, O_TOL, make_cross_inputs, softmax_scale

from gpu_helpers import compare_bwd, half_ulp

pytestmark = pytest.mark.gpu


def p8_of(p):
    return int(np.floor(p * 256 + 0.5))


def padding_mask(B, Sq, Sk, seed):
    """[B, 1, Sq, Sk_pad] uint8 key-padding storage (batch b sees its first L_b
    keys), rows padded to a multiple of 16 bytes; slice [..., :Sk] on the
    device to keep that row stride."""
    g = np.random.default_rng(seed)
    lens = g.integers(Sk // 3, Sk + 1, size=B)
    pad = (Sk + 15) // 16 * 16
    m = torch.zeros(B, 1, Sq, pad, dtype=torch.uint8)
    for b in range(B):
        m[b, :, :, :lens[b]] = 1
    return m


def bshd(t):
    return t.cuda().transpose(1, 2).contiguous().transpose(1, 2)


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("fp16", 64)])
def test_bshd_mask_dropout_forward_backward(causal, dtype, D):
    B, H, Sq, Sk, p = 2, 3, 200, 300, 0.15
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, dtype, seed=D + causal)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(3)).to(q.dtype)
    mask = padding_mask(B, Sq, Sk, 4)
    scale = softmax_scale(D)
    tq, tk, tv, tdo = (bshd(t) for t in (q, k, v, dout))
    dm = mask.cuda()[..., :Sk]  # a view of the padded storage: rows 16-byte aligned
    o = bshd(torch.empty(q.shape, dtype=q.dtype))
    o, lse = fa.flash_attention_forward(tq, tk, tv, scale, causal, out=o, dropout_p=p, seed=11, offset=5, mask=dm)
    gq, gk, gv = fa.flash_attention_backward(tq, tk, tv, o, lse, tdo, scale, causal, dropout_p=p, seed=11,
                                             offset=5, mask=dm)
    st = fa.fa_check_status(torch.cuda.current_stream().cuda_stream)
    assert st == 0, fa.fa_status_string(st)
    m_np = mask[..., :Sk].numpy()
    o_ref, lse_ref = oracle.attn_fwd_dropout(q, k, v, scale, causal, dtype, p8_of(p), 11, 5, mask=m_np)
    zs = 256.0 / (256.0 - p8_of(p))
    og = o.contiguous().cpu().double().numpy()
    err = np.abs(og - o_ref)
    rep = half_ulp(o_ref, dtype) < O_TOL[dtype] * zs
    assert err[rep].max() <= O_TOL[dtype] * zs
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= LSE_TOL
    refs = oracle.attn_bwd_dropout(q, k, v, dout, scale, causal, dtype, p8_of(p), 11, 5, magnitudes=True, mask=m_np)
    print(compare_bwd(tuple(t.contiguous().cpu() for t in (gq, gk, gv)), refs[:3], refs[3:], dtype, q, k, dout,
                      scale, causal))


def test_mask_and_keep_decisions_bit_exact():
    """V = identity over D keys: O[i, j] != 0 exactly where key j is visible
    (mask) and kept (dropout)."""
    B, H, S, D, p = 2, 2, 128, 128, 0.3
    q, k, _ = make_cross_inputs(B, H, S, S, D, "bf16", seed=9)
    v = torch.eye(D, dtype=torch.bfloat16).expand(B, H, D, D).contiguous()
    mask = padding_mask(B, S, S, 10)
    o, _ = fa.flash_attention_forward(q.cuda(), k.cuda(), v.cuda(), softmax_scale(D), False, dropout_p=p, seed=12,
                                      offset=13, mask=mask.cuda()[..., :S])
    torch.cuda.synchronize()
    keep = oracle.dropout_keep_mask(B * H, S, S, p8_of(p), 12, 13).reshape(B, H, S, S)
    want = keep.astype(bool) & mask[..., :S].numpy().astype(bool)
    assert np.array_equal(o.cpu().float().numpy() != 0, want)


def test_unified_entry_without_options_is_the_plain_kernel():
    q, k, v = make_cross_inputs(1, 2, 257, 300, 128, "bf16", seed=14)
    tq, tk, tv = (bshd(t) for t in (q, k, v))
    o1, l1 = fa.flash_attention_forward(tq, tk, tv, 0.1, True)          # fa_fwd_ex
    o2 = torch.empty_like(o1)
    l2 = torch.empty_like(l1)
    st = torch.cuda.current_stream().cuda_stream
    rc = fa.fa_forward(st, q=tq.data_ptr(), k=tk.data_ptr(), v=tv.data_ptr(), o=o2.data_ptr(), lse=l2.data_ptr(),
                       B=1, H=2, Sq=257, Sk=300, D=128, q_stride=tq.stride()[:3], k_stride=tk.stride()[:3],
                       v_stride=tv.stride()[:3], o_stride=o2.stride()[:3], scale=0.1, causal=1, dtype=fa.FA_BF16)
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)

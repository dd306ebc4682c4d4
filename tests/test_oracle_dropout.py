"""Pins of the oracle's attention dropout (attn_oracle.c, dropout section):
the Philox4x32-10 generator against its published known-answer vectors, the
keep rate, p = 0 giving the attention without dropout, the output written as
(P * keep / (1 - p)) V from the separately pinned probability matrix, the
unbiasedness of the estimate over offsets, and the gradients against float64
autograd of the same forward."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_18_b200.workloads import make_cross_inputs, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.json")


def test_philox_known_answer_vectors():
    with open(GOLDEN) as f:
        vecs = json.load(f)["vectors"]
    for v in vecs:
        ctr = [int(x, 16) for x in v["counter"]]
        key = [int(x, 16) for x in v["key"]]
        want = [int(x, 16) for x in v["output"]]
        assert list(oracle.philox4x32_10(ctr, key)) == want


def test_keep_mask_takes_bytes_of_the_counter_block():
    """Element j of row i uses byte j mod 16 of the block with counter (j / 16, i, bh, offset)."""
    seed, offset, p8 = 0x0123456789ABCDEF, 7, 100
    keep = oracle.dropout_keep_mask(3, 5, 40, p8, seed, offset)
    key = [seed & 0xffffffff, seed >> 32]
    for bh in range(3):
        for i in range(5):
            for g in range(3):
                w = oracle.philox4x32_10([g, i, bh, offset], key)
                by = np.frombuffer(w.astype("<u4").tobytes(), dtype=np.uint8)
                for b in range(16):
                    j = 16 * g + b
                    if j < 40:
                        assert keep[bh, i, j] == (by[b] >= p8)


@pytest.mark.parametrize("p8", [0, 26, 128, 255])
def test_keep_rate(p8):
    keep = oracle.dropout_keep_mask(2, 128, 512, p8, seed=12345, offset=0)
    n = keep.size
    rate = 1.0 - p8 / 256.0
    if p8 == 0:
        assert keep.all()
        return
    sigma = np.sqrt(rate * (1 - rate) / n)
    assert abs(keep.mean() - rate) < 5 * sigma


def test_offsets_and_seeds_give_different_masks():
    a = oracle.dropout_keep_mask(1, 64, 64, 128, seed=1, offset=0)
    b = oracle.dropout_keep_mask(1, 64, 64, 128, seed=1, offset=1)
    c = oracle.dropout_keep_mask(1, 64, 64, 128, seed=2, offset=0)
    assert (a != b).mean() > 0.4 and (a != c).mean() > 0.4


@pytest.mark.parametrize("causal", [False, True])
def test_p0_equals_attention_without_dropout(causal):
    q, k, v = make_cross_inputs(2, 2, 37, 53, 16, "bf16", seed=3)
    o0, l0 = oracle.attn_fwd_gen(q, k, v, 0.3, causal, "bf16")
    o1, l1 = oracle.attn_fwd_dropout(q, k, v, 0.3, causal, "bf16", 0, seed=99, offset=5)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)
    g = torch.Generator().manual_seed(4)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    r0 = oracle.attn_bwd(q, k, v, dout, 0.3, causal, "bf16")
    r1 = oracle.attn_bwd_dropout(q, k, v, dout, 0.3, causal, "bf16", 0, seed=99, offset=5)
    for a, b in zip(r0, r1):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("causal", [False, True])
def test_output_is_dropped_weights_times_v(causal):
    """O = (P * keep * 256 / (256 - p8)) V with P from attn_probs (pinned against
    SDPA) and keep from the generator; the LSE is the undropped one."""
    B, H, S, D, p8 = 1, 3, 40, 8, 77
    q, k, v = make_inputs(B, H, S, D, "fp16", seed=8)
    o, lse = oracle.attn_fwd_dropout(q, k, v, 0.5, causal, "fp16", p8, seed=5, offset=3)
    _, lse0 = oracle.attn_fwd(q, k, v, 0.5, causal, "fp16")
    assert np.array_equal(lse, lse0)
    keep = oracle.dropout_keep_mask(B * H, S, S, p8, 5, 3)
    vv = v.double().numpy()
    for bh in range(H):
        P = oracle.attn_probs(q, k, 0.5, causal, "fp16", bh=bh)
        want = (P * keep[bh] * (256.0 / (256.0 - p8))) @ vv[0, bh]
        assert np.allclose(o[0, bh], want, rtol=0, atol=1e-12)


def test_unbiased_over_offsets():
    """The mean of O over many dropout draws tends to the undropped O (within 5
    standard errors per element)."""
    q, k, v = make_inputs(1, 1, 8, 4, "bf16", seed=11)
    q = q * 3
    o_ref, _ = oracle.attn_fwd(q, k, v, 0.5, False, "bf16")
    n = 1500
    draws = np.stack([oracle.attn_fwd_dropout(q, k, v, 0.5, False, "bf16", 64, seed=21, offset=t)[0]
                      for t in range(n)])
    mean, se = draws.mean(0), draws.std(0) / np.sqrt(n)
    assert np.all(np.abs(mean - o_ref) <= 5 * se + 1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 2, 24, 24, 8), (2, 1, 17, 40, 16)])
def test_gradients_match_float64_autograd(causal, shape):
    B, H, Sq, Sk, D = shape
    p8, seed, offset, scale = 51, 77, 2, 0.375  # exact in float32, as the oracle takes it
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, "bf16", seed=Sq)
    g = torch.Generator().manual_seed(Sk)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    dq, dk, dv = oracle.attn_bwd_dropout(q, k, v, dout, scale, causal, "bf16", p8, seed, offset)
    keep = torch.from_numpy(oracle.dropout_keep_mask(B * H, Sq, Sk, p8, seed, offset).astype(np.float64))
    keep = keep.view(B, H, Sq, Sk)
    tq, tk, tv = (t.double().requires_grad_(True) for t in (q, k, v))
    s = scale * tq @ tk.transpose(-1, -2)
    if causal:
        i = torch.arange(Sq).view(-1, 1)
        j = torch.arange(Sk).view(1, -1)
        s = s.masked_fill(j > i + (Sk - Sq), float("-inf"))
    P = torch.softmax(s, dim=-1)
    o = (P * keep * (256.0 / (256.0 - p8))) @ tv
    (o * dout.double()).sum().backward()
    for name, mine, ref in (("dQ", dq, tq.grad), ("dK", dk, tk.grad), ("dV", dv, tv.grad)):
        assert np.allclose(mine, ref.numpy(), rtol=1e-10, atol=1e-12), name


def _padding_mask(B, Sq, Sk, seed):
    """A key-padding mask [B, 1, Sq, Sk]: batch b sees its first L_b keys."""
    g = np.random.default_rng(seed)
    lens = g.integers(Sk // 3, Sk + 1, size=B)
    m = np.zeros((B, 1, Sq, Sk), dtype=np.uint8)
    for b in range(B):
        m[b, :, :, :lens[b]] = 1
    return m


@pytest.mark.parametrize("causal", [False, True])
def test_mask_and_dropout_together(causal):
    """With a mask and dropout: an all-ones mask equals dropout alone and p8 = 0
    equals the mask alone (bitwise); O = (P_masked * keep * zs) V."""
    B, H, Sq, Sk, D, p8 = 2, 2, 24, 40, 8, 60
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, "bf16", seed=31)
    ones = np.ones((1, 1, Sq, Sk), dtype=np.uint8)
    a = oracle.attn_fwd_dropout(q, k, v, 0.5, causal, "bf16", p8, 3, 4)
    b = oracle.attn_fwd_dropout(q, k, v, 0.5, causal, "bf16", p8, 3, 4, mask=ones)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    m = _padding_mask(B, Sq, Sk, 5)
    c = oracle.attn_fwd_dropout(q, k, v, 0.5, causal, "bf16", 0, 3, 4, mask=m)
    d = oracle.attn_fwd_masked(q, k, v, m, 0.5, causal, "bf16")
    assert np.array_equal(c[0], d[0]) and np.array_equal(c[1], d[1])
    # the combination against its definition written with numpy
    o, lse = oracle.attn_fwd_dropout(q, k, v, 0.5, causal, "bf16", p8, 3, 4, mask=m)
    keep = oracle.dropout_keep_mask(B * H, Sq, Sk, p8, 3, 4).reshape(B, H, Sq, Sk)
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    s = 0.5 * qd @ kd.swapaxes(-1, -2)
    vis = np.broadcast_to(m.astype(bool), s.shape).copy()
    if causal:
        vis &= (np.arange(Sk)[None, :] <= np.arange(Sq)[:, None] + (Sk - Sq))
    s = np.where(vis, s, -np.inf)
    mx = s.max(-1, keepdims=True)
    p = np.exp(s - mx)
    l = p.sum(-1, keepdims=True)
    want = (p / l * keep * (256.0 / (256.0 - p8))) @ vd
    assert np.allclose(o, want, rtol=0, atol=1e-12)
    assert np.allclose(lse, (mx + np.log(l))[..., 0], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_mask_and_dropout_gradients_match_autograd(causal):
    B, H, Sq, Sk, D, p8, scale = 2, 2, 20, 33, 8, 77, 0.375
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, "fp16", seed=41)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(42)).to(torch.float16)
    m = _padding_mask(B, Sq, Sk, 6)
    dq, dk, dv = oracle.attn_bwd_dropout(q, k, v, dout, scale, causal, "fp16", p8, 8, 9, mask=m)
    keep = torch.from_numpy(oracle.dropout_keep_mask(B * H, Sq, Sk, p8, 8, 9).astype(np.float64)).view(B, H, Sq, Sk)
    tq, tk, tv = (t.double().requires_grad_(True) for t in (q, k, v))
    s = scale * tq @ tk.transpose(-1, -2)
    vis = torch.from_numpy(m.astype(bool)).expand(B, H, Sq, Sk)
    if causal:
        vis = vis & (torch.arange(Sk)[None, :] <= torch.arange(Sq)[:, None] + (Sk - Sq))
    s = s.masked_fill(~vis, float("-inf"))
    o = (torch.softmax(s, dim=-1) * keep * (256.0 / (256.0 - p8))) @ tv
    (o * dout.double()).sum().backward()
    for name, mine, ref in (("dQ", dq, tq.grad), ("dK", dk, tk.grad), ("dV", dv, tv.grad)):
        assert np.allclose(mine, ref.numpy(), rtol=1e-10, atol=1e-12), name


@pytest.mark.parametrize("Sq,Sk", [(70, 70), (40, 90), (90, 40)], ids=["square", "sq_lt_sk", "sq_gt_sk"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_sampled_rows_equal_full_run(Sq, Sk, causal):
    """The row-sampled dropout oracle (used by the GPU parity tests and the
    timed CPU baseline on large shapes) gives, bit for bit, the rows of the full
    dropout oracle: same keep decisions (the generator's counter takes the
    query row, not the sample index), same softmax and same scale.  The
    sample puts rows at positions other than their index, so a row/sample
    mix-up changes the keep decisions and fails."""
    from tiled_attention_18_b200.workloads import sample_rows
    if causal and Sq > Sk:
        pytest.skip("a causal query needs a key (Sq <= Sk)")
    B, H, D = 2, 3, 16
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, "bf16", seed=23)
    scale = 0.3
    for p8, seed, offset in ((26, 7, 0), (128, 0x123456789AB, 5), (255, 3, 2**32 - 1)):
        o, lse = oracle.attn_fwd_dropout(q, k, v, scale, causal, "bf16", p8, seed, offset)
        bh, rows = sample_rows(B, H, Sq, n_random=40, edge=3, seed=p8)
        assert not np.array_equal(rows, np.arange(rows.size) % Sq)
        orow, lrow = oracle.attn_rows_dropout(q, k, v, scale, causal, "bf16", p8, seed, offset, bh, rows)
        assert np.array_equal(orow, o.reshape(B * H, Sq, D)[bh, rows])
        assert np.array_equal(lrow, lse.reshape(B * H, Sq)[bh, rows])

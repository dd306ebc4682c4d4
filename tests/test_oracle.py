"""Pins for the fp64 CPU oracle (CPU only).

The oracle is pinned to things other than itself:
- a library routine that computes the same definition (torch SDPA and
  torch.logsumexp on the CPU in float64);
- a separately written tiled online-softmax recurrence (two forms);
- closed forms (Q = 0 gives the column mean / causal prefix mean of V and
  LSE = log of the key count; S = 1; constant V; hardmax at a large scale);
- invariants (softmax rows sum to 1, P V = O, key/value permutation);
- brute force (causal row i equals non-causal attention over keys 0..i; tile
  pairs counted element by element);
- the decoders against numpy float16 and torch bfloat16 on all 65,536 patterns;
- values the pages print (the causal tile table of the gsyq.cn catlass page).
A final group plants plausible mistakes in stand-in implementations and shows
that each one fails at least one of these pins.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_18_b200.workloads import make_inputs, softmax_scale

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

SMALL_SHAPES = [
    (1, 1, 1, 4), (1, 2, 2, 4), (2, 1, 5, 4), (1, 2, 17, 64), (2, 2, 64, 4), (1, 1, 130, 64),
]


def _f64(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.float64)


def _sdpa64(q, k, v, scale, causal):
    return torch.nn.functional.scaled_dot_product_attention(
        _f64(q), _f64(k), _f64(v), scale=float(scale), is_causal=bool(causal))


def _lse64(q, k, scale, causal):
    s = torch.matmul(_f64(q), _f64(k).transpose(-1, -2)) * float(scale)
    if causal:
        S = s.shape[-1]
        mask = torch.ones(S, S, dtype=torch.bool).triu(1)
        s = s.masked_fill(mask, float("-inf"))
    return torch.logsumexp(s, dim=-1)


# --------------------------------------------------------------- decoders

def test_f16_decoder_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode(bits, "fp16")
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_decoder_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.decode(bits, "bf16")
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


# ------------------------------------------------------ library reductions

@pytest.mark.parametrize("shape", SMALL_SHAPES)
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
def test_oracle_matches_sdpa_fp64(shape, dtype, causal):
    B, H, S, D = shape
    q, k, v = make_inputs(B, H, S, D, dtype, seed=S * 7 + D)
    scale = softmax_scale(D)
    o, lse = oracle.attn_fwd(q, k, v, scale, causal, dtype)
    ref = _sdpa64(q, k, v, scale, causal).numpy()
    assert np.max(np.abs(o - ref)) <= 1e-12
    ref_lse = _lse64(q, k, scale, causal).numpy()
    assert np.max(np.abs(lse - ref_lse)) <= 1e-12


def test_oracle_matches_sdpa_stressed_range():
    # Q, K x2 (the 13B-style workload's range) at a small size
    q, k, v = make_inputs(1, 2, 300, 128, "bf16", qk_mult=2.0, seed=3)
    scale = softmax_scale(128)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, scale, causal, "bf16")
        assert np.max(np.abs(o - _sdpa64(q, k, v, scale, causal).numpy())) <= 1e-12
        assert np.max(np.abs(lse - _lse64(q, k, scale, causal).numpy())) <= 1e-12


# ---------------------------------------------- tiled online recurrence

@pytest.mark.parametrize("S", [1, 2, 5, 17, 64, 130])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("form", [0, 1])
def test_tiled_reference_equals_naive(S, causal, form):
    q, k, v = make_inputs(2, 2, S, 4 if S < 64 else 64, "fp16", seed=S)
    D = q.shape[-1]
    scale = softmax_scale(D)
    o, lse = oracle.attn_fwd(q, k, v, scale, causal, "fp16")
    for br, bc in [(1, 1), (3, 7), (7, 3), (16, 16), (128, 128), (16, 128), (128, 16)]:
        ot, lt = oracle.attn_tiled(q, k, v, scale, causal, "fp16", br, bc, form)
        assert np.max(np.abs(ot - o)) <= 1e-12, (br, bc)
        assert np.max(np.abs(lt - lse)) <= 1e-12, (br, bc)


# --------------------------------------------------------- invariants

@pytest.mark.parametrize("causal", [False, True])
def test_softmax_rows_sum_to_one_and_pv_is_o(causal):
    q, k, v = make_inputs(1, 2, 40, 8, "bf16", seed=11)
    scale = softmax_scale(8)
    o, _ = oracle.attn_fwd(q, k, v, scale, causal, "bf16")
    vd = oracle.decode(oracle._bits(v), "bf16")
    for bh in range(2):
        p = oracle.attn_probs(q, k, scale, causal, "bf16", bh=bh)
        assert np.max(np.abs(p.sum(axis=1) - 1.0)) <= 1e-14
        assert np.all(p >= 0)
        if causal:
            assert np.all(np.triu(p, 1) == 0)
            assert np.all(np.diag(p) > 0)
        assert np.max(np.abs(p @ vd[0, bh] - o[0, bh])) <= 1e-13


def test_key_value_permutation_invariance():
    q, k, v = make_inputs(1, 1, 33, 16, "fp16", seed=5)
    scale = softmax_scale(16)
    o, lse = oracle.attn_fwd(q, k, v, scale, False, "fp16")
    perm = torch.randperm(33, generator=torch.Generator().manual_seed(9))
    o2, lse2 = oracle.attn_fwd(q, k[:, :, perm].contiguous(), v[:, :, perm].contiguous(), scale,
                               False, "fp16")
    assert np.max(np.abs(o - o2)) <= 1e-13
    assert np.max(np.abs(lse - lse2)) <= 1e-13


# --------------------------------------------------------- closed forms

@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_closed_form(dtype, causal):
    B, H, S, D = 1, 2, 37, 8
    _, k, v = make_inputs(B, H, S, D, dtype, seed=2)
    q = torch.zeros_like(k)
    o, lse = oracle.attn_fwd(q, k, v, 0.35, causal, dtype)
    vd = oracle.decode(oracle._bits(v), dtype)
    n = np.arange(1, S + 1, dtype=np.float64)
    if causal:
        ref = np.cumsum(vd, axis=2) / n[None, None, :, None]   # prefix mean of V
        ref_lse = np.broadcast_to(np.log(n), (B, H, S))
    else:
        ref = np.broadcast_to(vd.mean(axis=2, keepdims=True), vd.shape)  # column mean of V
        ref_lse = np.full((B, H, S), np.log(S))
    assert np.max(np.abs(o - ref)) <= 1e-14
    assert np.max(np.abs(lse - ref_lse)) <= 1e-14


def test_single_key_closed_form():
    q, k, v = make_inputs(2, 3, 1, 16, "bf16", seed=4)
    scale = softmax_scale(16)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, scale, causal, "bf16")
        qd = oracle.decode(oracle._bits(q), "bf16")
        kd = oracle.decode(oracle._bits(k), "bf16")
        vd = oracle.decode(oracle._bits(v), "bf16")
        assert np.array_equal(o, vd)
        ref = float(np.float32(scale)) * np.einsum("bhsd,bhsd->bhs", qd, kd)
        assert np.max(np.abs(lse - ref)) <= 1e-14


def test_constant_value_rows():
    q, k, _ = make_inputs(1, 2, 50, 8, "fp16", seed=6)
    v = torch.full_like(q, 1.5)
    o, _ = oracle.attn_fwd(q, k, v, softmax_scale(8), True, "fp16")
    assert np.max(np.abs(o - 1.5)) <= 1e-14


def test_hardmax_at_large_scale():
    # distinct scores and a huge scale: each row selects V at its argmax score
    B, H, S, D = 1, 1, 24, 8
    q, k, v = make_inputs(B, H, S, D, "fp16", seed=8)
    scale = 1.0e4
    o, _ = oracle.attn_fwd(q, k, v, scale, False, "fp16")
    s = (_f64(q) @ _f64(k).transpose(-1, -2))[0, 0].numpy()
    srt = np.sort(s, axis=1)
    assert np.all(srt[:, -1] - srt[:, -2] > 0.01), "scores must be distinct for this check"
    arg = s.argmax(axis=1)
    vd = oracle.decode(oracle._bits(v), "fp16")[0, 0]
    assert np.max(np.abs(o[0, 0] - vd[arg])) <= 1e-12


# --------------------------------------------------------- brute force

@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_causal_row_equals_prefix_attention(dtype):
    B, H, S, D = 1, 2, 29, 16
    q, k, v = make_inputs(B, H, S, D, dtype, seed=12)
    scale = softmax_scale(D)
    o, lse = oracle.attn_fwd(q, k, v, scale, True, dtype)
    for i in range(S):
        qi = q[:, :, i:i + 1].contiguous()
        oi, li = oracle.attn_fwd(qi.expand(B, H, i + 1, D).contiguous(),
                                 k[:, :, :i + 1].contiguous(), v[:, :, :i + 1].contiguous(),
                                 scale, False, dtype)
        assert np.max(np.abs(o[:, :, i] - oi[:, :, 0])) <= 1e-14
        assert np.max(np.abs(lse[:, :, i] - li[:, :, 0])) <= 1e-14


def test_sampled_rows_equal_full_run():
    from tiled_attention_18_b200.workloads import sample_rows
    B, H, S, D = 2, 3, 70, 16
    q, k, v = make_inputs(B, H, S, D, "bf16", seed=21)
    scale = softmax_scale(D)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, scale, causal, "bf16")
        bh, rows = sample_rows(B, H, S, n_random=50)
        orow, lrow = oracle.attn_rows(q, k, v, scale, causal, "bf16", bh, rows)
        ofl = o.reshape(B * H, S, D)
        assert np.array_equal(orow, ofl[bh, rows])
        assert np.array_equal(lrow, lse.reshape(B * H, S)[bh, rows])


def _loop_bound_computed(S, BM, BN):
    """Pairs visited by the diagonal loop bound j <= floor(((m+1)*BM - 1) / BN)."""
    nq, nk = -(-S // BM), -(-S // BN)
    return sum(min(((m + 1) * BM - 1) // BN + 1, nk) for m in range(nq))


@pytest.mark.parametrize("BM,BN", [(64, 64), (128, 128), (128, 64), (64, 128), (256, 128)])
def test_causal_tile_enumeration_matches_loop_bound(BM, BN):
    for S in list(range(1, 300)) + [511, 512, 513, 1000, 1024]:
        total, computed, skipped = oracle.causal_tile_count(S, BM, BN)
        nq, nk = -(-S // BM), -(-S // BN)
        assert total == nq * nk
        assert computed + skipped == total
        assert computed == _loop_bound_computed(S, BM, BN), (S, BM, BN)


def test_causal_tile_table_from_page():
    with open(os.path.join(GOLDEN, "causal_skip_table.json")) as f:
        g = json.load(f)
    BM, BN = g["tile"]
    for row in g["rows"]:
        total, computed, skipped = oracle.causal_tile_count(row["S"], BM, BN)
        T = row["S"] // BM
        assert total == row["total"]                   # printed total is exact
        assert skipped == T * (T - 1) // 2             # exact count strictly above the diagonal
        assert computed == T * (T + 1) // 2
        # the printed count is the rounded half; within one diagonal of tiles of it
        assert abs(skipped - row["skipped_printed"]) <= T
        assert abs(skipped / total - row["ratio_printed"]) <= 1.0 / T


def test_worked_example_shapes():
    with open(os.path.join(GOLDEN, "ops_transformer_shapes.json")) as f:
        g = json.load(f)
    # same B, H, D and causal flag at a shorter sequence (the oracle's cost is S^2)
    S = 64
    q, k, v = make_inputs(g["B"], g["H"], S, g["D"], "fp16", seed=0)
    o, lse = oracle.attn_fwd(q, k, v, softmax_scale(g["D"]), g["causal"], "fp16")
    printed = g["output_shape_printed"]
    assert list(o.shape) == [printed[0], printed[1], S, printed[3]]
    assert lse.shape == (g["B"], g["H"], S)


# --------------------------------------- planted mistakes fail the pins

def _np_attention(q, k, v, scale, causal, mistake=None):
    """Stand-in numpy attention with one planted mistake (mistake=None is correct)."""
    q, k, v = (_f64(x).numpy() for x in (q, k, v))
    S = q.shape[2]
    s = np.einsum("bhid,bhjd->bhij", q, k)
    if mistake == "scale_sqrt":
        s = s * np.sqrt(scale)
    elif mistake != "no_scale":
        s = s * scale
    keep = np.ones((S, S), bool)
    if causal:
        if mistake == "strict_causal":        # j < i instead of j <= i (row 0 keeps key 0)
            keep = np.tril(keep, -1)
            keep[0, 0] = True
        elif mistake == "upper_causal":        # the mask on the wrong side
            keep = np.triu(keep)
        else:
            keep = np.tril(keep)
    if mistake == "drop_last_key":            # a ragged tail that loses the last key
        keep[:, S - 1] = False
        keep[S - 1, S - 1] = causal and keep[S - 1, S - 2]
    s = np.where(keep, s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    axis = -2 if mistake == "softmax_wrong_axis" else -1
    l = e.sum(axis=axis, keepdims=True)
    if mistake == "no_normalise":
        l = np.ones_like(l)
    p = e / l
    vv = k if mistake == "k_for_v" else v
    o = np.einsum("bhij,bhjd->bhid", p, vv)
    lsum = e.sum(axis=-1)
    if mistake == "lse_log2":
        lse = m[..., 0] / np.log(2) + np.log2(lsum)
    elif mistake == "lse_no_max":
        lse = np.log(lsum)
    else:
        lse = m[..., 0] + np.log(lsum)
    return o, lse


def _pins_pass(impl) -> bool:
    """Run the value pins (SDPA fp64, logsumexp, Q=0 closed form, causal prefix) on impl."""
    try:
        for causal in (False, True):
            q, k, v = make_inputs(1, 2, 12, 4, "fp16", seed=31)
            scale = softmax_scale(4)
            o, lse = impl(q, k, v, scale, causal)
            if np.max(np.abs(o - _sdpa64(q, k, v, scale, causal).numpy())) > 1e-12:
                return False
            if np.max(np.abs(lse - _lse64(q, k, scale, causal).numpy())) > 1e-12:
                return False
            q0 = torch.zeros_like(q)
            o0, l0 = impl(q0, k, v, 0.5, causal)
            vd = _f64(v).numpy()
            n = np.arange(1, 13, dtype=np.float64)
            ref = (np.cumsum(vd, axis=2) / n[None, None, :, None]) if causal else \
                np.broadcast_to(vd.mean(axis=2, keepdims=True), vd.shape)
            if np.max(np.abs(o0 - ref)) > 1e-12:
                return False
    except Exception:
        return False
    return True


def test_pins_accept_the_oracle_and_a_correct_standin():
    assert _pins_pass(lambda q, k, v, s, c: oracle.attn_fwd(q, k, v, s, c, "fp16"))
    assert _pins_pass(lambda q, k, v, s, c: _np_attention(q, k, v, s, c))


@pytest.mark.parametrize("mistake", ["no_scale", "scale_sqrt", "strict_causal", "upper_causal",
                                     "softmax_wrong_axis", "no_normalise", "lse_log2",
                                     "lse_no_max", "drop_last_key", "k_for_v"])
def test_pins_reject_planted_mistakes(mistake):
    assert not _pins_pass(lambda q, k, v, s, c: _np_attention(q, k, v, s, c, mistake))

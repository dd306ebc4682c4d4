"""Pins for the backward-pass oracle (CPU only).

The gradients are checked against: float64 autograd through an explicit
attention (softmax of masked scaled scores times V); central finite
differences of the forward oracle (a separate code path: no derivative
formula involved); closed forms (constant V gives dQ = dK = 0 and
dV_j = sum_i P_ij dO_i; a single key gives dQ = dK = 0, dV = sum of dO); and the
identities sum_j dK_j = 0 (the Jacobian rows of a softmax sum to zero) and
sum_j dV_j = sum_i dO_i (each P row sums to one).
"""
import numpy as np
import pytest
import torch

import oracle
from tiled_attention_18_b200.workloads import make_cross_inputs, make_inputs


def _dout(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    t = torch.randn(shape, generator=g, dtype=torch.float32)
    return t.to(torch.float16 if dtype == "fp16" else torch.bfloat16)


def _autograd_ref(q, k, v, dout, scale, causal):
    q64, k64, v64 = (t.to(torch.float64).requires_grad_(True) for t in (q, k, v))
    s = torch.matmul(q64, k64.transpose(-1, -2)) * float(np.float32(scale))
    if causal:
        Sq, Sk = q.shape[2], k.shape[2]
        i = torch.arange(Sq)[:, None]
        j = torch.arange(Sk)[None, :]
        s = s.masked_fill(j > i + (Sk - Sq), float("-inf"))
    o = torch.matmul(torch.softmax(s, dim=-1), v64)
    o.backward(dout.to(torch.float64))
    return q64.grad.numpy(), k64.grad.numpy(), v64.grad.numpy()


@pytest.mark.parametrize("Sq,Sk", [(1, 1), (5, 5), (33, 33), (7, 40), (40, 7), (64, 130)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_bwd_matches_fp64_autograd(Sq, Sk, causal, dtype):
    if causal and Sq > Sk:
        pytest.skip("rows without keys: checked separately")
    q, k, v = make_cross_inputs(2, 2, Sq, Sk, 16, dtype, seed=Sq + 3 * Sk)
    dout = _dout(q.shape, dtype, seed=Sq * Sk + 1)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, 0.3, causal, dtype)
    rq, rk, rv = _autograd_ref(q, k, v, dout, 0.3, causal)
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.max(np.abs(a - b)) <= 1e-12 * max(1.0, np.max(np.abs(b)))


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_matches_central_differences_of_the_forward_oracle(causal):
    """<dO, dF/dx . E> by central differences of attn_fwd_gen, for every input
    element of a tiny problem; the forward oracle takes 16-bit inputs, so the
    perturbation is applied to an fp64 copy through a float16-exact scaling:
    we differentiate L(t) = <dO, O(x + t e)> with t = +-h on inputs that stay
    exactly representable (x and e chosen on a coarse grid)."""
    B, H, Sq, Sk, D = 1, 1, 4, 6, 4
    rng = np.random.default_rng(7)
    # values on a grid of 1/8 in [-2, 2]: exact in fp16, and x +- h (h = 1/256) too
    grid = lambda shape: (rng.integers(-16, 17, size=shape) / 8.0)  # noqa: E731
    q, k, v = (torch.tensor(grid((B, H, n, D)), dtype=torch.float16) for n in (Sq, Sk, Sk))
    dout = torch.tensor(grid((B, H, Sq, D)), dtype=torch.float16)
    scale = 0.5
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, scale, causal, "fp16")
    h = 1.0 / 256
    g = dout.to(torch.float64).numpy()

    def loss(qq, kk, vv):
        o, _ = oracle.attn_fwd_gen(qq, kk, vv, scale, causal, "fp16")
        return float((o * g).sum())

    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in np.ndindex(*x.shape):
            xp, xm = x.clone(), x.clone()
            xp[idx] += h
            xm[idx] -= h
            assert float(xp[idx]) - float(x[idx]) == h  # exact in fp16
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            fd = (loss(args_p["q"], args_p["k"], args_p["v"]) - loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
            assert abs(fd - grad[idx]) <= 2e-4 * max(1.0, abs(grad[idx])), (name, idx, fd, grad[idx])


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_constant_values_closed_form(causal):
    q, k, v = make_inputs(1, 2, 24, 8, "bf16", seed=5)
    v = v[:, :, :1].expand(v.shape).contiguous()          # every v_j equal
    dout = _dout(q.shape, "bf16", seed=6)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, 0.4, causal, "bf16")
    assert np.max(np.abs(dq)) <= 1e-13 and np.max(np.abs(dk)) <= 1e-13
    # dV_j = sum_i P_ij dO_i with the forward oracle's softmax matrix
    for h in range(2):
        probs = oracle.attn_probs(q, k, 0.4, causal, "bf16", bh=h)
        ref = probs.T @ dout[0, h].to(torch.float64).numpy()
        assert np.max(np.abs(dv[0, h] - ref)) <= 1e-12


def test_bwd_single_key():
    q, k, v = make_cross_inputs(1, 3, 9, 1, 16, "fp16", seed=8)
    dout = _dout(q.shape, "fp16", seed=9)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, 0.25, False, "fp16")
    assert np.max(np.abs(dq)) <= 1e-14 and np.max(np.abs(dk)) <= 1e-14
    assert np.max(np.abs(dv[:, :, 0] - dout.to(torch.float64).numpy().sum(axis=2))) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_column_sum_identities(causal):
    q, k, v = make_inputs(2, 2, 77, 32, "bf16", seed=10)
    dout = _dout(q.shape, "bf16", seed=11)
    dq, dk, dv, mq, mk, mv = oracle.attn_bwd(q, k, v, dout, 0.2, causal, "bf16", magnitudes=True)
    assert np.max(np.abs(dk.sum(axis=2))) <= 1e-11 * max(1.0, np.max(np.abs(dk)))
    assert np.max(np.abs(dv.sum(axis=2) - dout.to(torch.float64).numpy().sum(axis=2))) <= 1e-11
    # the magnitudes bound the gradients element by element
    for g, m in ((dq, mq), (dk, mk), (dv, mv)):
        assert np.all(np.abs(g) <= m * (1 + 1e-12) + 1e-300)


def test_bwd_rows_without_keys_get_no_gradient():
    q, k, v = make_cross_inputs(1, 1, 10, 4, 8, "fp16", seed=12)   # Sq > Sk, causal: rows 0..5 see nothing
    dout = _dout(q.shape, "fp16", seed=13)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, 0.5, True, "fp16")
    assert np.all(dq[0, 0, :6] == 0)
    rq, rk, rv = _autograd_ref(q[:, :, 6:], k, v, dout[:, :, 6:], 0.5, True)   # the other rows alone
    assert np.max(np.abs(dq[:, :, 6:] - rq)) <= 1e-12
    assert np.max(np.abs(dk - rk)) <= 1e-12 and np.max(np.abs(dv - rv)) <= 1e-12


# --------------------------------------- planted mistakes fail the pins

def _np_bwd(q, k, v, dout, scale, causal, mistake=None):
    """Stand-in numpy backward (square, top-left causal) with one planted mistake."""
    q, k, v, g = (x.to(torch.float64).numpy() for x in (q, k, v, dout))
    scale = float(np.float32(scale))   # the callers' scale is a float32 value
    S = q.shape[2]
    s = np.einsum("bhid,bhjd->bhij", q, k) * scale
    if causal:
        s = np.where(np.tril(np.ones((S, S), bool)), s, -np.inf)
    p = np.exp(s - s.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    dp = np.einsum("bhid,bhjd->bhij", g, v)
    if mistake == "dsum_unweighted":
        dsum = dp.sum(-1, keepdims=True)
    else:
        dsum = (p * dp).sum(-1, keepdims=True)
    ds = p * dp if mistake == "no_dsum" else p * (dp - dsum)
    dq = np.einsum("bhij,bhjd->bhid", ds, v if mistake == "dq_uses_v" else k) * scale
    dk = np.einsum("bhij,bhid->bhjd", ds, q) * (1.0 if mistake == "dk_no_scale" else scale)
    if mistake == "dv_no_transpose":
        dv = np.einsum("bhij,bhjd->bhid", p, g)
    elif mistake == "dv_uses_ds":
        dv = np.einsum("bhij,bhid->bhjd", ds, g)
    else:
        dv = np.einsum("bhij,bhid->bhjd", p, g)
    return dq, dk, dv


def _bwd_pins_pass(impl) -> bool:
    try:
        for causal in (False, True):
            q, k, v = make_inputs(1, 2, 12, 4, "bf16", seed=41)
            dout = _dout(q.shape, "bf16", seed=42)
            dq, dk, dv = impl(q, k, v, dout, 0.4, causal)
            rq, rk, rv = _autograd_ref(q, k, v, dout, 0.4, causal)
            if max(np.max(np.abs(dq - rq)), np.max(np.abs(dk - rk)), np.max(np.abs(dv - rv))) > 1e-12:
                return False
            if np.max(np.abs(dk.sum(axis=2))) > 1e-12:
                return False
            if np.max(np.abs(dv.sum(axis=2) - dout.to(torch.float64).numpy().sum(axis=2))) > 1e-12:
                return False
    except Exception:
        return False
    return True


def test_bwd_pins_accept_the_oracle_and_a_correct_standin():
    assert _bwd_pins_pass(lambda q, k, v, g, s, c: oracle.attn_bwd(q, k, v, g, s, c, "bf16"))
    assert _bwd_pins_pass(lambda q, k, v, g, s, c: _np_bwd(q, k, v, g, s, c))


@pytest.mark.parametrize("mistake", ["no_dsum", "dsum_unweighted", "dq_uses_v", "dk_no_scale",
                                     "dv_no_transpose", "dv_uses_ds"])
def test_bwd_pins_reject_planted_mistakes(mistake):
    assert not _bwd_pins_pass(lambda q, k, v, g, s, c: _np_bwd(q, k, v, g, s, c, mistake))

"""GPU parity of the backward pass on short key sets, whose (head, key tile)
work units leave SMs idle: the query range of the key tile is then split into
chunks across units, each adding its share of dK and dV in fp32 to the
workspace before one conversion kernel writes them (D = 64, 128 and 256;
split without an explicit mask or dropout for D = 128/256, with them for
D = 64).  Every gradient element is compared with the fp64 oracle within the
suite's backward bound; deterministic mode (no split) must still repeat bit
for bit.
"""
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import GENERAL_WORKLOADS, make_cross_inputs, softmax_scale, workload_inputs

from gpu_helpers import compare_bwd, run_fa_bwd

pytestmark = pytest.mark.gpu


def _dout(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.float16 if dtype == "fp16" else torch.bfloat16)


SHAPES = [
    # (B, H, Sq, Sk, D, causal): few heads, one key tile, several query steps
    (1, 1, 1000, 77, 64, False), (1, 2, 640, 128, 64, False), (1, 1, 300, 17, 128, False),
    (1, 2, 513, 100, 128, False), (1, 1, 120, 128, 128, True), (1, 1, 500, 64, 256, False),
    (2, 3, 700, 33, 64, False), (1, 1, 129, 1, 64, False),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_short_key_backward_matches_oracle(shape, dtype):
    B, H, Sq, Sk, D, causal = shape
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, dtype, seed=3 * Sq + Sk)
    dout = _dout(q.shape, dtype, seed=Sq + 5 * Sk)
    scale = softmax_scale(D)
    gq, gk, gv, _, _ = run_fa_bwd(q, k, v, dout, scale, causal)
    dq, dk, dv, mq, mk, mv = oracle.attn_bwd(q, k, v, dout, scale, causal, dtype, magnitudes=True)
    print(shape, dtype, compare_bwd((gq, gk, gv), (dq, dk, dv), (mq, mk, mv), dtype, q, k, dout, scale, causal))


def test_sdxl_cross_attention_backward_full_compare():
    """2 x 10 heads, 4096 image-token queries over 77 text-token keys, D = 64, fp16."""
    w = GENERAL_WORKLOADS["sdxl_xattn"]
    q, k, v = workload_inputs(w)
    dout = _dout(q.shape, w.dtype, seed=77)
    gq, gk, gv, _, _ = run_fa_bwd(q, k, v, dout, w.scale, w.causal)
    dq, dk, dv, mq, mk, mv = oracle.attn_bwd(q, k, v, dout, w.scale, w.causal, w.dtype, magnitudes=True)
    compare_bwd((gq, gk, gv), (dq, dk, dv), (mq, mk, mv), w.dtype, q, k, dout, w.scale, w.causal)


@pytest.mark.parametrize("D", [64, 128])
def test_short_key_deterministic_backward_repeats_bitwise(D):
    q, k, v = make_cross_inputs(1, 2, 700, 77, D, "bf16", seed=D)
    dout = _dout(q.shape, "bf16", seed=D + 1)
    scale = softmax_scale(D)
    runs = [run_fa_bwd(q, k, v, dout, scale, False, deterministic=True)[:3] for _ in range(2)]
    for a, b in zip(*runs):
        assert torch.equal(a, b)
    dq, dk, dv, mq, mk, mv = oracle.attn_bwd(q, k, v, dout, scale, False, "bf16", magnitudes=True)
    compare_bwd(runs[0], (dq, dk, dv), (mq, mk, mv), "bf16", q, k, dout, scale, False)


@pytest.mark.parametrize("D", [64, 128])
def test_short_key_masked_backward(D):
    """The explicit mask (D = 64: split query range; D = 128: one unit per key tile)."""
    B, H, Sq, Sk = 1, 2, 600, 77
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, "bf16", seed=21 + D)
    dout = _dout(q.shape, "bf16", seed=22 + D)
    scale = softmax_scale(D)
    g = torch.Generator().manual_seed(23)
    mask = torch.rand((1, H, Sq, Sk), generator=g) < 0.7
    mask[..., :, 0] = True
    dq_, dk_, dv_, ddo = (t.cuda() for t in (q, k, v, dout))
    pad = -(-Sk // 16) * 16
    mbuf = torch.zeros((1, H, Sq, pad), dtype=torch.uint8)
    mbuf[..., :Sk] = mask.to(torch.uint8)
    dm = mbuf.cuda()[..., :Sk]
    o, lse = fa.flash_attention_forward(dq_, dk_, dv_, scale, False, mask=dm)
    grads = fa.flash_attention_backward(dq_, dk_, dv_, o, lse, ddo, scale, False, mask=dm)
    assert fa.fa_check_status(torch.cuda.current_stream().cuda_stream) == 0
    refs = oracle.attn_bwd_masked(q, k, v, dout, mask, scale, False, "bf16", magnitudes=True)
    compare_bwd(tuple(t.cpu() for t in grads), refs[:3], refs[3:], "bf16", q, k, dout, scale, False)

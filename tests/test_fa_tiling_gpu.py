"""Manual tilings of the forward kernel (fa_forward's block_n and q_tiles):
key tiles of 64 or 128 rows, one or two 128-row query tiles per work unit.
Every tiling computes the same attention; each is compared element by
element with the fp64 oracle on ragged shapes, with and without the causal
mask, and the default tiling given explicitly equals fa_fwd bit for bit."""
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import make_cross_inputs, make_inputs, softmax_scale

from gpu_helpers import compare

pytestmark = pytest.mark.gpu

TILINGS = [(64, 1), (64, 2), (128, 1), (128, 2)]


@pytest.mark.parametrize("block_n,q_tiles", TILINGS, ids=lambda x: str(x))
@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("fp16", 64), ("fp16", 128), ("bf16", 64)])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("S", [1, 63, 130, 300, 777])
def test_tiling_matches_oracle(block_n, q_tiles, dtype, D, causal, S):
    B, H = 1, 2
    q, k, v = make_inputs(B, H, S, D, dtype, seed=4000 + S)
    scale = softmax_scale(D)
    o, lse = fa.flash_attention_forward(q.cuda(), k.cuda(), v.cuda(), scale, causal, block_n=block_n,
                                        q_tiles=q_tiles)
    assert fa.fa_check_status(torch.cuda.current_stream().cuda_stream) == 0
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, scale, causal, dtype)
    compare(o.cpu(), lse.cpu(), o_ref, lse_ref, dtype)


@pytest.mark.parametrize("block_n,q_tiles", TILINGS, ids=lambda x: str(x))
@pytest.mark.parametrize("Sq,Sk,causal", [(200, 77, False), (300, 1000, True), (513, 600, False)])
def test_tiling_cross_shapes(block_n, q_tiles, Sq, Sk, causal):
    q, k, v = make_cross_inputs(2, 3, Sq, Sk, 128, "bf16", seed=71)
    scale = softmax_scale(128)
    o, lse = fa.flash_attention_forward(q.cuda(), k.cuda(), v.cuda(), scale, causal, block_n=block_n,
                                        q_tiles=q_tiles)
    o_ref, lse_ref = oracle.attn_fwd_gen(q, k, v, scale, causal, "bf16")
    compare(o.cpu(), lse.cpu(), o_ref, lse_ref, "bf16")


def test_default_tiling_given_explicitly_is_fa_fwd():
    q, k, v = (t.cuda() for t in make_inputs(1, 3, 1000, 128, "bf16", seed=3))
    for causal in (False, True):
        o_ref, lse_ref = fa.flash_attention_forward(q, k, v, 0.1, causal)
        o, lse = fa.flash_attention_forward(q, k, v, 0.1, causal, block_n=128, q_tiles=2)
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)

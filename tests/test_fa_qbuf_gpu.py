"""GPU parity of the D = 64 forward with two Q buffers, against the fp64 oracle,
through the C ABI.

Without an explicit mask or dropout, a D = 64 launch whose CTAs run two or
more work units each (units >= 2 x grid) uses the instantiation with two Q
buffers: the next unit's Q loads while the current unit runs, and the next
unit's first S product is issued before the current unit's last P.V.  The
shapes cover ragged query and key counts, units whose second query tile is
empty (Sq <= 128), cross-attention with the bottom-right causal mask, both
16-bit types, and a BSHD layout written in place; every shape has at least
two units per CTA on a 148-SM B200.
"""
import pytest

import oracle
from tiled_attention_18_b200.workloads import make_cross_inputs, softmax_scale

from gpu_helpers import compare, run_fa_ex

pytestmark = pytest.mark.gpu

SHAPES = [
    # (B, H, Sq, Sk): units = B * H * ceil(Sq / 256)
    (4, 40, 1000, 1000),   # 640 units, ragged tail tiles
    (2, 160, 100, 300),    # 320 units, the second query tile of every unit empty
    (3, 50, 300, 700),     # 300 units, cross-attention (Sq < Sk)
    (1, 300, 256, 129),    # 300 units, one full key tile and one key in the second
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_two_q_buffers_match_oracle(shape, dtype, causal):
    B, H, Sq, Sk = shape
    if causal and Sq > Sk:
        pytest.skip("causal needs Sq <= Sk")
    q, k, v = make_cross_inputs(B, H, Sq, Sk, 64, dtype, seed=7 * Sq + Sk)
    scale = softmax_scale(64)
    o, lse = run_fa_ex(q, k, v, scale, causal)
    o_ref, lse_ref = oracle.attn_fwd_gen(q, k, v, scale, causal, dtype)
    compare(o, lse, o_ref, lse_ref, dtype)


def test_two_q_buffers_bshd_in_place():
    B, H, S = 8, 40, 512
    q, k, v = make_cross_inputs(B, H, S, S, 64, "fp16", seed=5)
    scale = softmax_scale(64)
    o, lse = run_fa_ex(q, k, v, scale, False, layouts=("bshd",) * 4)
    o_ref, lse_ref = oracle.attn_fwd_gen(q, k, v, scale, False, "fp16")
    compare(o, lse, o_ref, lse_ref, "fp16")

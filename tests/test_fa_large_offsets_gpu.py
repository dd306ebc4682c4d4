"""Element offsets beyond 2^31: every tensor of a forward and a backward call
lives in one buffer with a head stride above 2^31 elements (the second head
starts past 2^31), so tensor-map coordinates, the O/LSE epilogue, the
backward's prep kernel and its gradient stores all index beyond 32 bits.
Small S keeps the work tiny; results are compared with the fp64 oracle on
contiguous copies."""
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import make_inputs, softmax_scale

from gpu_helpers import compare, compare_bwd

pytestmark = pytest.mark.gpu

HEAD_STRIDE = 2**31 + 4096  # elements; a multiple of 8


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_forward_and_backward_past_2_pow_31(causal):
    B, H, S, D, dtype = 1, 2, 600, 128, "bf16"
    q, k, v = make_inputs(B, H, S, D, dtype, seed=21)
    g = torch.Generator().manual_seed(22)
    dout = torch.randn(q.shape, generator=g).to(q.dtype)
    slot = S * D
    buf = torch.zeros(HEAD_STRIDE + 9 * slot, dtype=q.dtype, device="cuda")  # about 4.3 GB

    def view(i):  # tensor i of the call: slot i of each head's region
        return buf[i * slot:].as_strided((B, H, S, D), (H * HEAD_STRIDE, HEAD_STRIDE, D, 1))

    tq, tk, tv, to, tdo, gq, gk, gv = (view(i) for i in range(8))
    for dst, src in ((tq, q), (tk, k), (tv, v), (tdo, dout)):
        dst.copy_(src.cuda())
    scale = softmax_scale(D)
    o, lse = fa.flash_attention_forward(tq, tk, tv, scale, causal, out=to)
    fa.flash_attention_backward(tq, tk, tv, o, lse, tdo, scale, causal, dq=gq, dk=gk, dv=gv)
    st = fa.fa_check_status(torch.cuda.current_stream().cuda_stream)
    assert st == 0, fa.fa_status_string(st)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, scale, causal, dtype)
    compare(o.contiguous().cpu(), lse.cpu(), o_ref, lse_ref, dtype)
    refs = oracle.attn_bwd(q, k, v, dout, scale, causal, dtype, magnitudes=True)
    compare_bwd(tuple(t.contiguous().cpu() for t in (gq, gk, gv)), refs[:3], refs[3:], dtype, q, k, dout, scale,
                causal)
    # nothing was written outside the eight slots of the two heads
    for h in range(H):
        lo = h * HEAD_STRIDE + 8 * slot
        assert not buf[lo:lo + slot].any()
    del buf
    torch.cuda.empty_cache()

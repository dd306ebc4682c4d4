"""``attention`` (forward + backward through autograd) on the GPU against the
fp64 oracle's gradients."""
import numpy as np
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import make_cross_inputs

from gpu_helpers import compare_bwd

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dropout", [0.0, 0.2], ids=["plain", "dropout"])
def test_attention_autograd_matches_oracle(dropout):
    B, H, Sq, Sk, D = 1, 2, 200, 300, 128
    q, k, v = make_cross_inputs(B, H, Sq, Sk, D, "bf16", seed=51)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(52)).to(torch.bfloat16)
    tq, tk, tv = (t.cuda().requires_grad_(True) for t in (q, k, v))
    o = fa.attention(tq, tk, tv, scale=0.09, causal=True, dropout_p=dropout, seed=3, offset=4)
    (o * dout.cuda()).sum().backward()
    assert fa.fa_check_status(torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    if dropout:
        p8 = int(np.floor(dropout * 256 + 0.5))
        refs = oracle.attn_bwd_dropout(q, k, v, dout, 0.09, True, "bf16", p8, 3, 4, magnitudes=True)
    else:
        refs = oracle.attn_bwd(q, k, v, dout, 0.09, True, "bf16", magnitudes=True)
    compare_bwd((tq.grad.cpu(), tk.grad.cpu(), tv.grad.cpu()), refs[:3], refs[3:], "bf16", q, k, dout, 0.09, True)

"""Back-to-back launches on one stream read what the launch before them wrote.

Every kernel is a programmatic dependent launch: it may start while the
previous kernel in the stream is still running and waits (griddepcontrol.wait)
before its first global-memory access.  These tests chain launches whose
inputs are the previous launch's outputs, with no host synchronisation in
between, on output buffers pre-filled with a value that would show in the
result if a launch read them early: each stage must equal the fp64 oracle
applied to the previous stage's final output.  The chains cover the short-key,
streaming (D = 64 with one and two Q buffers, D = 128) and D = 256 forward
kernels, a forward followed by the three backward kernels, and the same chain
captured in a CUDA graph and replayed.
"""
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import make_cross_inputs, softmax_scale

from gpu_helpers import compare, compare_bwd

pytestmark = pytest.mark.gpu

POISON = 3.0e4

CHAINS = [
    # (B, H, S, Sk, D): S queries over Sk keys; Q of each stage = O of the one before
    (2, 10, 1024, 77, 64),     # short-key kernel
    (1, 8, 1000, 1000, 64),    # streaming kernel, one Q buffer
    (4, 40, 512, 512, 64),     # streaming kernel, two Q buffers (>= 2 units per CTA)
    (2, 16, 700, 900, 128),    # streaming kernel, D = 128
    (1, 4, 500, 600, 256),     # D = 256 kernel
]


def _chain(q, k, v, scale, causal, n, outs, lses):
    x = q
    for i in range(n):
        fa.flash_attention_forward(x, k, v, scale, causal, out=outs[i], lse=lses[i])
        x = outs[i]


@pytest.mark.parametrize("shape", CHAINS, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("graph", [False, True], ids=["stream", "graph"])
def test_forward_chain_reads_final_outputs(shape, graph):
    B, H, S, Sk, D = shape
    dtype, n = "bf16", 3
    causal = Sk >= S
    q, k, v = make_cross_inputs(B, H, S, Sk, D, dtype, seed=S + D)
    # scale up so that each stage's output differs clearly from its input
    q = (q.float() * 4).to(q.dtype)
    scale = softmax_scale(D)
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    outs = [torch.full_like(dq, POISON) for _ in range(n)]
    lses = [torch.full((B, H, S), POISON, dtype=torch.float32, device="cuda") for _ in range(n)]
    if graph:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            _chain(dq, dk, dv, scale, causal, n, outs, lses)
        torch.cuda.current_stream().wait_stream(s)
        for t in outs:
            t.fill_(POISON)
        g.replay()
    else:
        _chain(dq, dk, dv, scale, causal, n, outs, lses)
    torch.cuda.synchronize()
    assert fa.fa_check_status(torch.cuda.current_stream().cuda_stream) == 0
    x = q
    for i in range(n):
        o_ref, lse_ref = oracle.attn_fwd_gen(x, k, v, scale, causal, dtype)
        compare(outs[i].cpu(), lses[i].cpu(), o_ref, lse_ref, dtype)
        x = outs[i].cpu()


@pytest.mark.parametrize("D", [64, 128])
def test_backward_right_after_forward(D):
    """Forward, then the backward's prep, main and post kernels, then a second
    forward on dQ: no synchronisation anywhere in between."""
    B, H, S = 2, 4, 384
    dtype = "fp16"
    q, k, v = make_cross_inputs(B, H, S, S, D, dtype, seed=D)
    g = torch.Generator().manual_seed(3)
    do = torch.randn(q.shape, generator=g).to(q.dtype)
    scale = softmax_scale(D)
    dq_, dk_, dv_, ddo = (t.cuda() for t in (q, k, v, do))
    o = torch.full_like(dq_, POISON)
    lse = torch.full((B, H, S), POISON, dtype=torch.float32, device="cuda")
    grads = [torch.full_like(dq_, POISON) for _ in range(3)]
    o2 = torch.full_like(dq_, POISON)
    lse2 = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, S, D), dtype=torch.uint8, device="cuda")
    fa.flash_attention_forward(dq_, dk_, dv_, scale, True, out=o, lse=lse)
    fa.flash_attention_backward(dq_, dk_, dv_, o, lse, ddo, scale, True, dq=grads[0], dk=grads[1], dv=grads[2],
                                workspace=ws)
    fa.flash_attention_forward(grads[0], dk_, dv_, scale, True, out=o2, lse=lse2)
    torch.cuda.synchronize()
    assert fa.fa_check_status(torch.cuda.current_stream().cuda_stream) == 0
    o_ref, lse_ref = oracle.attn_fwd_gen(q, k, v, scale, True, dtype)
    compare(o.cpu(), lse.cpu(), o_ref, lse_ref, dtype)
    dq, dk, dv, mq, mk, mv = oracle.attn_bwd(q, k, v, do, scale, True, dtype, magnitudes=True)
    compare_bwd([t.cpu() for t in grads], (dq, dk, dv), (mq, mk, mv), dtype, q, k, do, scale, True)
    o2_ref, lse2_ref = oracle.attn_fwd_gen(grads[0].cpu(), k, v, scale, True, dtype)
    compare(o2.cpu(), lse2.cpu(), o2_ref, lse2_ref, dtype)

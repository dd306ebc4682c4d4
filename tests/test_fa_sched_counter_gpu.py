"""Causal launches of different grid sizes and kernels, back to back on one stream.

A causal forward launch takes its work units from a per-stream counter (units
claimed longest first); the last CTA of each launch clears the counter and its
count of finished CTAs, so the next causal launch on the stream starts from
zero with nothing run in between.  These tests chain causal launches whose
grids differ (a handful of CTAs, then one per SM, then a handful again), whose
kernels differ (D = 64, 128 and 256 share the stream's counter), and whose
shapes include cross-attention with the bottom-right mask, with no host
synchronisation anywhere in the chain; each output must equal the fp64 oracle.
The same chain is then captured in a CUDA graph and replayed twice, which
checks that a replay finds the counter cleared by the replay before it.
"""
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import make_cross_inputs, softmax_scale

from gpu_helpers import compare

pytestmark = pytest.mark.gpu

POISON = 3.0e4

CHAIN = [
    # (B, H, Sq, Sk, D, dtype): units = B * H * ceil(Sq / 256); grid = min(units, SMs)
    (1, 2, 300, 300, 128, "bf16"),     # 4 units: 4 CTAs
    (1, 20, 2048, 2048, 128, "fp16"),  # 160 units: one CTA per SM
    (1, 3, 700, 700, 64, "fp16"),      # 9 units
    (1, 4, 600, 600, 256, "bf16"),     # the D = 256 kernel, same counter
    (4, 40, 512, 512, 64, "bf16"),     # 320 units: one CTA per SM, two or more units each
    (2, 3, 200, 900, 128, "fp16"),     # cross-attention, bottom-right causal mask
    (1, 2, 300, 300, 128, "bf16"),     # the first launch again
]


def _inputs():
    ins = []
    for i, (B, H, Sq, Sk, D, dtype) in enumerate(CHAIN):
        q, k, v = make_cross_inputs(B, H, Sq, Sk, D, dtype, seed=100 + i)
        ins.append((q, k, v, tuple(t.cuda() for t in (q, k, v))))
    return ins


def _launch_all(ins, outs, lses):
    for (shape, (_, _, _, (dq, dk, dv)), o, lse) in zip(CHAIN, ins, outs, lses):
        fa.flash_attention_forward(dq, dk, dv, softmax_scale(shape[4]), True, out=o, lse=lse)


def _check(ins, outs, lses):
    assert fa.fa_check_status(torch.cuda.current_stream().cuda_stream) == 0
    for (shape, (q, k, v, _), o, lse) in zip(CHAIN, ins, outs, lses):
        dtype = shape[5]
        o_ref, lse_ref = oracle.attn_fwd_gen(q, k, v, softmax_scale(shape[4]), True, dtype)
        compare(o.cpu(), lse.cpu(), o_ref, lse_ref, dtype)


def _buffers(ins):
    outs = [torch.full_like(dev[0], POISON) for (_, _, _, dev) in ins]
    lses = [torch.full(dev[0].shape[:3], POISON, dtype=torch.float32, device="cuda") for (_, _, _, dev) in ins]
    return outs, lses


def test_causal_chain_on_one_stream():
    ins = _inputs()
    outs, lses = _buffers(ins)
    for _ in range(2):  # the second pass starts from the counter the first pass left
        for t in outs:
            t.fill_(POISON)
        _launch_all(ins, outs, lses)
        torch.cuda.synchronize()
        _check(ins, outs, lses)


def test_causal_chain_graph_replayed():
    ins = _inputs()
    outs, lses = _buffers(ins)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        _launch_all(ins, outs, lses)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(2):
        for t in outs:
            t.fill_(POISON)
        g.replay()
        torch.cuda.synchronize()
        _check(ins, outs, lses)

"""The library's calls inside CUDA graphs: forward and backward captured once
(after a warm-up call on the capture stream, which allocates the causal
scheduler's counter) and replayed with new inputs copied into the captured
buffers give the same bits as eager calls (deterministic dQ order)."""
import pytest
import torch

import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import make_inputs, softmax_scale

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("fp16", 64)])
def test_forward_backward_graph_replay(causal, dtype, D):
    B, H, S = 1, 4, 640
    scale = softmax_scale(D)
    inputs = [make_inputs(B, H, S, D, dtype, seed=s) for s in (1, 2, 3)]
    douts = [torch.randn(inputs[0][0].shape, generator=torch.Generator().manual_seed(10 + s)).to(inputs[0][0].dtype)
             for s in range(3)]
    sq, sk, sv = (t.cuda() for t in inputs[0])
    sdo = douts[0].cuda()
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, S, D), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())

    def step():
        o, lse = fa.flash_attention_forward(sq, sk, sv, scale, causal)
        grads = fa.flash_attention_backward(sq, sk, sv, o, lse, sdo, scale, causal, deterministic=True, workspace=ws)
        return (o, lse) + grads

    with torch.cuda.stream(stream):
        step()  # warm-up on the capture stream
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        outs = step()
    for (q, k, v), dout in zip(inputs, douts):
        for dst, src in ((sq, q), (sk, k), (sv, v), (sdo, dout)):
            dst.copy_(src)
        graph.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in outs]
        want = step()
        torch.cuda.synchronize()
        assert fa.fa_check_status(torch.cuda.current_stream().cuda_stream) == 0
        for name, a, b in zip(("o", "lse", "dq", "dk", "dv"), got, want):
            assert torch.equal(a, b), name

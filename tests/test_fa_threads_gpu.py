"""Forward calls from several host threads at once, on one stream."""
import threading

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.mark.xfail(strict=False, reason="before launches returned their own status and the shared-memory "
                   "limit was set once per kernel, two of four threads got FA_ERR_LAUNCH here; "
                   "the change has not yet run on a B200")
def test_causal_calls_from_several_threads_on_one_stream():
    """Four threads issue causal forwards on torch's default stream at the same
    time.  Each call's scheduler-counter reset and launch stay together, so
    every call computes all its rows (checked against the oracle)."""
    import tiled_attention_18_b200 as fa
    from tiled_attention_18_b200.workloads import O_TOL, make_inputs, softmax_scale
    n = 4
    inputs = [make_inputs(1, 4, 1024, 128, "bf16", seed=100 + i) for i in range(n)]
    dev = [tuple(t.cuda() for t in x) for x in inputs]
    outs = [None] * n
    errors = []
    start = threading.Barrier(n)

    def work(i):
        try:
            start.wait(timeout=60)
            for _ in range(5):
                outs[i] = fa.flash_attention_forward(*dev[i], softmax_scale(128), True)
        except Exception as e:  # reported below, with the thread's index
            errors.append((i, repr(e)))

    threads = [threading.Thread(target=work, args=(i,)) for i in range(n)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    torch.cuda.synchronize()
    assert not errors, errors
    assert fa.fa_check_status(torch.cuda.current_stream().cuda_stream) == 0
    for i in range(n):
        o_ref, _ = oracle.attn_fwd(*inputs[i], softmax_scale(128), True, "bf16")
        assert np.abs(outs[i][0].cpu().double().numpy() - o_ref).max() <= O_TOL["bf16"]

"""Forward calls from several host threads at once, on one stream and on a
stream per thread."""
import threading

import pytest
import torch

import oracle

from gpu_helpers import compare

pytestmark = pytest.mark.gpu


def _run_threads(n, per_thread_stream):
    """n threads issue causal forwards at the same time; each thread's
    exceptions carry the CUDA error the library recorded for that thread."""
    import tiled_attention_18_b200 as fa
    from tiled_attention_18_b200.workloads import make_inputs, softmax_scale
    inputs = [make_inputs(1, 4, 1024, 128, "bf16", seed=100 + i) for i in range(n)]
    dev = [tuple(t.cuda() for t in x) for x in inputs]
    streams = [torch.cuda.Stream() if per_thread_stream else None for _ in range(n)]
    torch.cuda.synchronize()
    outs = [None] * n
    errors = []
    start = threading.Barrier(n)

    def work(i):
        try:
            start.wait(timeout=60)
            for _ in range(5):
                outs[i] = fa.flash_attention_forward(*dev[i], softmax_scale(128), True, stream=streams[i])
        except Exception as e:  # reported below, with the thread's index and its CUDA error record
            errors.append((i, repr(e), fa.fa_last_cuda_error()))

    threads = [threading.Thread(target=work, args=(i,)) for i in range(n)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    torch.cuda.synchronize()
    assert not errors, errors
    for s in streams:
        assert fa.fa_check_status(s.cuda_stream if s is not None else torch.cuda.current_stream().cuda_stream) == 0
    for i in range(n):
        o, lse = outs[i]
        o_ref, lse_ref = oracle.attn_fwd(*inputs[i], softmax_scale(128), True, "bf16")
        compare(o.cpu(), lse.cpu(), o_ref, lse_ref, "bf16")


def test_causal_calls_from_several_threads_on_one_stream():
    """Four threads issue causal forwards on torch's default stream at the same
    time.  Each call's scheduler-counter reset and launch stay together, so
    every call computes all its rows (checked against the oracle)."""
    _run_threads(4, per_thread_stream=False)


def test_causal_calls_from_several_threads_on_own_streams():
    """Four threads, each on a stream of its own: every stream gets its own
    scheduler counter, so the kernels may overlap on the GPU."""
    _run_threads(4, per_thread_stream=True)

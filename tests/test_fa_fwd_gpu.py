"""GPU parity of fa_fwd (through the C ABI) against the fp64 CPU oracle.

- small and ragged shapes, both head dims, both dtypes, with and without the
  causal mask: every output element against the oracle;
- the workload configurations, every output element against the full fp64
  oracle, the long-sequence ones (S = 8192, 16384) in the launch
  configuration the benchmark times;
- properties that hold at any size: Q = 0 gives the column mean / causal
  prefix mean of V and LSE = log(key count); causal row 0 equals V_0;
- bitwise determinism across runs, and every output row written.
"""
import json
import math

import numpy as np
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import WORKLOADS, make_inputs, softmax_scale, workload_inputs

from gpu_helpers import compare, run_fa

pytestmark = pytest.mark.gpu


SMALL = [
    # (B, H, S, D)
    (1, 1, 1, 64), (1, 1, 17, 128), (1, 2, 127, 64), (1, 1, 128, 128), (1, 3, 129, 64),
    (2, 1, 255, 128), (1, 2, 256, 64), (1, 1, 257, 128), (2, 3, 300, 64), (1, 2, 513, 128),
    (1, 1, 640, 64),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_small_shapes_match_oracle(shape, dtype, causal):
    B, H, S, D = shape
    q, k, v = make_inputs(B, H, S, D, dtype, seed=1000 + S + D)
    scale = softmax_scale(D)
    o, lse = run_fa(q, k, v, scale, causal)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, scale, causal, dtype)
    compare(o, lse, o_ref, lse_ref, dtype)


@pytest.mark.parametrize("name", ["c1", "c2", "c3"])
def test_workload_full_compare(name):
    w = WORKLOADS[name]
    q, k, v = workload_inputs(w)
    o, lse = run_fa(q, k, v, w.scale, w.causal)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, w.scale, w.causal, w.dtype)
    r = compare(o, lse, o_ref, lse_ref, w.dtype)
    print("parity", name, json.dumps(r))


@pytest.mark.parametrize("name", ["c4", "c5a", "c5b"])
def test_workload_long_full_compare(name):
    """The long-sequence workloads (S = 8192 and 16384), every output element
    against the full fp64 oracle, in the launch configuration the benchmark
    times (the oracle takes minutes of host time here, all cores)."""
    w = WORKLOADS[name]
    q, k, v = workload_inputs(w)
    o, lse = run_fa(q, k, v, w.scale, w.causal)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()  # every row written (outputs started as NaN)
    if w.causal:
        # row 0 attends to key 0 only: O_0 = V_0 exactly
        assert torch.equal(o[:, :, 0], v[:, :, 0])
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, w.scale, w.causal, w.dtype)
    r = compare(o, lse, o_ref, lse_ref, w.dtype)
    print("parity", name, json.dumps(r))


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("S,D", [(1000, 64), (4096, 128)])
def test_zero_query_closed_form(dtype, causal, S, D):
    B, H = 1, 2
    _, k, v = make_inputs(B, H, S, D, dtype, seed=77)
    q = torch.zeros_like(k)
    o, lse = run_fa(q, k, v, 0.125, causal)
    vd = v.to(torch.float64).numpy()
    n = np.arange(1, S + 1, dtype=np.float64)
    if causal:
        ref = np.cumsum(vd, axis=2) / n[None, None, :, None]
        ref_lse = np.broadcast_to(np.log(n), (B, H, S))
    else:
        ref = np.broadcast_to(vd.mean(axis=2, keepdims=True), vd.shape)
        ref_lse = np.full((B, H, S), math.log(S))
    compare(o, lse, ref, ref_lse, dtype)


def test_deterministic_and_stream():
    w = WORKLOADS["c3"]
    q, k, v = (t.cuda() for t in workload_inputs(w))
    s = torch.cuda.Stream()
    outs = []
    with torch.cuda.stream(s):
        for _ in range(3):
            o, lse = fa.flash_attention_forward(q, k, v, w.scale, w.causal)
            outs.append((o.clone(), lse.clone()))
    s.synchronize()
    assert fa.fa_check_status(s.cuda_stream) == 0
    for o, lse in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(lse, outs[0][1])


@pytest.mark.parametrize("D", [128, 256])
def test_causal_call_on_a_new_stream_allocates_nothing(D):
    """The causal scheduler's counter comes from a static pool in the library:
    the first causal fa_fwd on a stream the library has not seen before leaves
    the device's free memory unchanged, and two streams running at once keep
    separate counters (both results match a single-stream run bit for bit)."""
    q, k, v = (t.cuda() for t in make_inputs(1, 4, 1500, D, "bf16", seed=31))
    scale = softmax_scale(D)
    o_ref, lse_ref = fa.flash_attention_forward(q, k, v, scale, True)  # kernels loaded
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [(torch.empty_like(q), torch.empty((1, 4, 1500), dtype=torch.float32, device="cuda")) for _ in streams]
    for s in streams:
        with torch.cuda.stream(s):
            outs[0][0].zero_()  # each stream's first launch is not the library's
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for s, (o, lse) in zip(streams, outs):
        fa.flash_attention_forward(q, k, v, scale, True, out=o, lse=lse, stream=s)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before, f"device free memory moved by {free_before - free_after} bytes"
    for s in streams:
        assert fa.fa_check_status(s.cuda_stream) == 0
    for o, lse in outs:
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_scale_is_honoured():
    q, k, v = make_inputs(1, 2, 200, 64, "fp16", seed=5)
    for scale in (0.01, 0.125, 0.7):
        o, lse = run_fa(q, k, v, scale, False)
        o_ref, lse_ref = oracle.attn_fwd(q, k, v, scale, False, "fp16")
        compare(o, lse, o_ref, lse_ref, "fp16")


def test_host_side_errors_on_device():
    q = torch.zeros((1, 1, 64, 64), dtype=torch.float16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, 64), dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    ok = fa.fa_fwd(q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(), lse.data_ptr(), 1, 1, 64, 64,
                   0.125, 0, fa.FA_FP16, st)
    assert ok == 0
    # misaligned pointer
    assert fa.fa_fwd(q.data_ptr() + 2, q.data_ptr(), q.data_ptr(), o.data_ptr(), lse.data_ptr(), 1, 1, 64, 64,
                     0.125, 0, fa.FA_FP16, st) == -5
    # host memory is rejected before any launch
    host = torch.zeros((1, 1, 64, 64), dtype=torch.float16).pin_memory()
    assert fa.fa_fwd(host.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(), lse.data_ptr(), 1, 1, 64, 64,
                     0.125, 0, fa.FA_FP16, st) == -11
    # empty problem: nothing launched, pointers not inspected
    assert fa.fa_fwd(0, 0, 0, 0, 0, 0, 4, 64, 64, 0.125, 0, fa.FA_FP16, st) == 0
    assert fa.fa_check_status(st) == 0


def test_stuck_wait_reports_timeout_and_context_survives():
    """A wait that nothing satisfies ends with FA_ERR_TIMEOUT (no hang, no fault),
    and the library keeps working afterwards."""
    st = torch.cuda.current_stream().cuda_stream
    assert fa.fa_check_status(st) == 0
    assert fa.fa_selftest_timeout(st) == 0
    assert fa.fa_check_status(st) == -8           # FA_ERR_TIMEOUT
    assert fa.fa_last_timeout_site() & 0xFF == 100
    assert fa.fa_check_status(st) == 0            # the status word was cleared
    q, k, v = make_inputs(1, 2, 300, 64, "fp16", seed=9)
    o, lse = run_fa(q, k, v, softmax_scale(64), True)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, softmax_scale(64), True, "fp16")
    compare(o, lse, o_ref, lse_ref, "fp16")


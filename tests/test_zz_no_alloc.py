"""fa_fwd_noalloc: the entry point for callers that cannot allocate device
memory (its scratch is a fixed array inside the library).  It must give the
same results as fa_fwd, call after call (the array keeps the previous call's
contents, so each call has to clear what it relies on), and it must not
change the device's free memory, even on a stream that no call of the
library has used before.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.workloads import LSE_TOL, O_TOL, make_inputs, softmax_scale

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,D,causal", [("bf16", 128, True), ("fp16", 64, True), ("bf16", 128, False),
                                            ("bf16", 256, True)])
def test_noalloc_matches_fa_fwd_on_two_calls_in_a_row(dtype, D, causal):
    fa.load()
    B, H, S = 2, 3, 1000
    q, k, v = (t.cuda() for t in make_inputs(B, H, S, D, dtype, seed=321))
    scale = softmax_scale(D)
    code = fa.FA_BF16 if dtype == "bf16" else fa.FA_FP16
    st0 = torch.cuda.current_stream().cuda_stream

    o_ref = torch.empty_like(q)
    lse_ref = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    assert fa.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o_ref.data_ptr(), lse_ref.data_ptr(),
                     B, H, S, D, scale, int(causal), code, st0) == 0
    # one call on the default stream first: the library's kernels and its static
    # array are loaded (lazy module loading) before free memory is measured
    o = torch.empty_like(q)
    lse = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    assert fa.fa_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                             B, H, S, D, scale, int(causal), code, st0) == 0

    # a stream the library has never seen, outputs allocated up front
    fresh = torch.cuda.Stream()
    outs = [(torch.full_like(q, float("nan")), torch.full((B, H, S), float("nan"), dtype=torch.float32,
                                                          device="cuda")) for _ in range(2)]
    with torch.cuda.stream(fresh):
        outs[0][0].fill_(float("nan"))  # the stream's first launch is not the library's
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for o, lse in outs:
        rc = fa.fa_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                               B, H, S, D, scale, int(causal), code, fresh.cuda_stream)
        assert rc == 0, fa.fa_status_string(rc)
    fresh.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before, f"device free memory moved by {free_before - free_after} bytes"
    assert fa.fa_check_status(fresh.cuda_stream) == 0

    for call, (o, lse) in enumerate(outs):
        do = (o.double() - o_ref.double()).abs().max().item()
        dl = (lse.double() - lse_ref.double()).abs().max().item()
        assert np.isfinite(do) and do <= O_TOL[dtype], f"call {call}: max |dO| {do}"
        assert np.isfinite(dl) and dl <= LSE_TOL, f"call {call}: max |dLSE| {dl}"


def test_noalloc_rejects_bad_arguments_like_fa_fwd():
    fa.load()
    # argument errors are found before any device work, as in fa_fwd
    assert fa.fa_fwd_noalloc(0, 0, 0, 0, 0, 1, 1, 128, 96, 0.1, 0, 0, 0) == -3   # head dim
    assert fa.fa_fwd_noalloc(0, 0, 0, 0, 0, 0, 1, 128, 64, 0.1, 1, 0, 0) == 0    # empty problem

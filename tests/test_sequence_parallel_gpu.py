"""Sequence-parallel attention through the library's kernels on one GPU: the
ring and all-gather schedules of every rank of a W-rank group are run in one
process (the K/V block each rank would receive is handed to it directly), and
the concatenated result is compared with the fp64 oracle's full attention.
Covers fa_merge_partial / fa_merge_finalize and the block-causal logic; the
P2P/all-gather communication itself is covered by the gloo tests."""
import numpy as np
import pytest
import torch

import oracle
import tiled_attention_18_b200 as fa
from tiled_attention_18_b200.sequence_parallel import CudaOps, allgather_attention_forward, ring_attention_forward
from tiled_attention_18_b200.workloads import make_inputs, softmax_scale

from gpu_helpers import compare

pytestmark = pytest.mark.gpu


def _run_all_ranks(mode, q, k, v, world, scale, causal):
    B, H, S, D = q.shape
    c = S // world
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    chunks = [(dq[:, :, r * c:(r + 1) * c].contiguous(), dk[:, :, r * c:(r + 1) * c].contiguous(),
               dv[:, :, r * c:(r + 1) * c].contiguous()) for r in range(world)]
    kv_blocks = [torch.stack([ck, cv]) for (_, ck, cv) in chunks]
    outs, lses = [], []
    for r in range(world):
        qr, kr, vr = chunks[r]
        ops = CudaOps(scale)
        if mode == "ring":
            # at step s the rank holds rank (r - s)'s block and receives rank (r - s - 1)'s
            o, lse = ring_attention_forward(qr, kr, vr, scale, causal, ops=ops, rank=r, world=world,
                                            exchange=lambda s, kv, r=r: (None, kv_blocks[(r - s - 1) % world]))
        else:
            o, lse = allgather_attention_forward(qr, kr, vr, scale, causal, ops=ops, rank=r, world=world,
                                                 gather=lambda kv: torch.stack(kv_blocks))
        outs.append(o)
        lses.append(lse)
    st = torch.cuda.current_stream().cuda_stream
    assert fa.fa_check_status(st) == 0
    torch.cuda.synchronize()
    return torch.cat(outs, dim=2).cpu(), torch.cat(lses, dim=2).cpu()


@pytest.mark.parametrize("mode", ["ring", "allgather"])
@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("fp16", 64)])
def test_sequence_parallel_schedules_match_full_attention(mode, world, causal, dtype, D):
    q, k, v = make_inputs(1, 4, 1024, D, dtype, seed=world + D)
    scale = softmax_scale(D)
    o, lse = _run_all_ranks(mode, q, k, v, world, scale, causal)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, scale, causal, dtype)
    print(mode, world, causal, dtype, compare(o, lse, o_ref, lse_ref, dtype))


def test_merge_partial_matches_union_and_empty_sides():
    """Two disjoint key halves merged equal attention over all keys; an empty
    partial (LSE = -inf) leaves the running result unchanged."""
    q, k, v = make_inputs(2, 3, 384, 128, "bf16", seed=7)
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    ops = CudaOps(0.09)
    state = ops.init(dq)
    for lo, hi in ((0, 200), (200, 384)):
        o_p, lse_p = fa.flash_attention_forward(dq, dk[:, :, lo:hi].contiguous(), dv[:, :, lo:hi].contiguous(), 0.09)
        ops.merge(state, o_p, lse_p)
    before = state[0].clone(), state[1].clone()
    empty_o = torch.zeros_like(dq)
    empty_l = torch.full(dq.shape[:3], float("-inf"), device="cuda")
    ops.merge(state, empty_o, empty_l)
    assert torch.equal(state[0], before[0]) and torch.equal(state[1], before[1])
    o, lse = ops.finalize(state)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, 0.09, False, "bf16")
    compare(o.cpu(), lse.cpu(), o_ref, lse_ref, "bf16")


@pytest.mark.parametrize("D,offset", [(128, 0), (64, 0), (98, 0), (128, 1)], ids=["d128", "d64", "d98", "unaligned"])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_merge_partial_kernel_matches_fp64_merge(D, offset, dtype):
    """fa_merge_partial against the log-sum-exp combination written out in
    fp64, with rows where either side or both sides are empty (LSE = -inf);
    D = 98 and a buffer offset by one element take the scalar variant."""
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    rows = 1000
    g = torch.Generator().manual_seed(D + offset)
    o_acc = torch.randn(rows * D + offset, generator=g)
    l_acc = torch.randn(rows, generator=g) * 4
    o_p = torch.randn(rows * D + offset, generator=g).to(tdt)
    l_p = torch.randn(rows, generator=g) * 4
    l_acc[::7] = float("-inf")
    l_p[::11] = float("-inf")
    a0 = o_acc[offset:].view(rows, D).double().numpy()
    b0 = o_p[offset:].view(rows, D).double().numpy()
    la, lb = l_acc.double().numpy(), l_p.double().numpy()
    m = np.maximum(la, lb)
    with np.errstate(invalid="ignore"):
        wa = np.where(np.isinf(la), 0.0, np.exp(la - m))
        wb = np.where(np.isinf(lb), 0.0, np.exp(lb - m))
        s = wa + wb
        o_ref = np.where((s > 0)[:, None], (wa[:, None] * a0 + wb[:, None] * b0) / np.where(s > 0, s, 1)[:, None], a0)
        l_ref = np.where(s > 0, m + np.log(np.where(s > 0, s, 1)), la)
    d_acc, d_lacc, d_p, d_lp = (t.cuda() for t in (o_acc, l_acc, o_p, l_p))
    rc = fa.fa_merge_partial(d_acc.data_ptr() + 4 * offset, d_lacc.data_ptr(), d_p.data_ptr() + 2 * offset,
                             d_lp.data_ptr(), rows, D, 1 if dtype == "bf16" else 0,
                             torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    got_o = d_acc.cpu()[offset:].view(rows, D).double().numpy()
    got_l = d_lacc.cpu().double().numpy()
    # fp32 weights and products: a few ulps of fp32 relative to the row's magnitude
    scale_o = np.abs(a0).max(axis=1, keepdims=True) + np.abs(b0).max(axis=1, keepdims=True)
    assert np.all(np.abs(got_o - o_ref) <= 4e-6 * scale_o)
    both_empty = np.isinf(la) & np.isinf(lb)
    assert np.all(np.isneginf(got_l[both_empty]))
    assert np.all(np.abs(got_l[~both_empty] - l_ref[~both_empty]) <= 4e-6 * (1 + np.abs(l_ref[~both_empty])))


def test_merge_finalize_rounds_to_nearest_even():
    x = torch.randn(4099, generator=torch.Generator().manual_seed(3)) * 10
    for tdt, code in ((torch.bfloat16, 1), (torch.float16, 0)):
        dx = x.cuda()
        out = torch.empty(4099, dtype=tdt, device="cuda")
        assert fa.fa_merge_finalize(dx.data_ptr(), out.data_ptr(), 4099, code,
                                    torch.cuda.current_stream().cuda_stream) == 0
        torch.cuda.synchronize()
        assert torch.equal(out.cpu(), x.to(tdt))


def _run_ranks_in_threads(world, fn):
    """fn(rank, exchange) for every rank, each in its own thread; exchange hands a
    payload to rank + 1 and returns the one from rank - 1.  All threads launch on
    the same CUDA stream, so the launch order orders the work."""
    import queue
    import threading
    boxes = [queue.Queue() for _ in range(world)]
    results, errors = [None] * world, []

    def make_exchange(r):
        def exchange(step, payload):
            boxes[(r + 1) % world].put(payload)
            return None, boxes[r].get(timeout=120)
        return exchange

    def body(r):
        try:
            results[r] = fn(r, make_exchange(r))
        except Exception as e:  # re-raised in the test thread
            errors.append(e)

    threads = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    if errors:
        raise errors[0]
    return results


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("fp16", 64)])
def test_ring_backward_through_the_kernels(world, causal, dtype, D):
    """Every rank's ring backward (fa_bwd partials for the global O and LSE,
    fa_accumulate, fa_merge_finalize) on one GPU; the gathered gradients against
    the oracle's gradients over the whole sequence.  Each rank rounds its 16-bit
    partials once before the fp32 sums and the sums once at the end: together at
    most 2 more units of u * mag than one fa_bwd call, hence the bound c = 4."""
    from gpu_helpers import compare_bwd
    from tiled_attention_18_b200.sequence_parallel import ring_attention_backward
    B, H, S = 1, 3, 512
    c = S // world
    q, k, v = make_inputs(B, H, S, D, dtype, seed=world + D)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(5)).to(q.dtype)
    scale = softmax_scale(D)
    dq, dk, dv, ddo = (t.cuda() for t in (q, k, v, dout))
    o, lse = fa.flash_attention_forward(dq, dk, dv, scale, causal)  # the forward's global rows
    part = lambda t, r: t[:, :, r * c:(r + 1) * c].contiguous()  # noqa: E731

    def rank_fn(r, exchange):
        return ring_attention_backward(part(dq, r), part(dk, r), part(dv, r), part(o, r), part(lse, r),
                                       part(ddo, r), scale, causal, ops=CudaOps(scale), exchange=exchange, rank=r,
                                       world=world)

    res = _run_ranks_in_threads(world, rank_fn)
    assert fa.fa_check_status(torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    grads = tuple(torch.cat([res[r][i] for r in range(world)], dim=2).cpu() for i in range(3))
    refs = oracle.attn_bwd(q, k, v, dout, scale, causal, dtype, magnitudes=True)
    print(compare_bwd(grads, refs[:3], refs[3:], dtype, q, k, dout, scale, causal, c=4.0))


def test_accumulate_kernel():
    for tdt, code, n in ((torch.bfloat16, 1, 4096), (torch.float16, 0, 1001)):
        x = torch.randn(n, generator=torch.Generator().manual_seed(n)).to(tdt)
        acc0 = torch.randn(n, generator=torch.Generator().manual_seed(n + 1))
        dacc, dx = acc0.cuda(), x.cuda()
        assert fa.fa_accumulate(dacc.data_ptr(), dx.data_ptr(), n, code, torch.cuda.current_stream().cuda_stream) == 0
        torch.cuda.synchronize()
        assert torch.equal(dacc.cpu(), acc0 + x.float())


class _ThreadAllToAll:
    """all-to-all among threads: rank r's x[p] goes to rank p, which gets them
    stacked by source rank.  Two barriers per call: all have written, all
    have read."""

    def __init__(self, world):
        import threading
        self.world = world
        self.slots = [[None] * world for _ in range(world)]
        self.barrier = threading.Barrier(world)

    def make(self, r):
        def a2a(x):
            for p in range(self.world):
                self.slots[p][r] = x[p]
            self.barrier.wait(timeout=120)
            out = torch.stack([self.slots[r][p] for p in range(self.world)])
            self.barrier.wait(timeout=120)
            return out
        return a2a


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("fp16", 64)])
def test_ulysses_through_the_kernels(world, causal, dtype, D):
    """Head-parallel forward and backward, every rank in its own thread on one
    GPU: the kernels run on whole heads, so the results are those of single
    calls on the full sequence (forward tolerance; backward bound of fa_bwd)."""
    from gpu_helpers import compare, compare_bwd
    from tiled_attention_18_b200.sequence_parallel import ulysses_attention_backward, ulysses_attention_forward
    B, H, S = 1, 4, 512
    c = S // world
    q, k, v = make_inputs(B, H, S, D, dtype, seed=world + 2 * D)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(6)).to(q.dtype)
    scale = softmax_scale(D)
    dq, dk, dv, ddo = (t.cuda() for t in (q, k, v, dout))
    part = lambda t, r: t[:, :, r * c:(r + 1) * c].contiguous()  # noqa: E731
    comm = _ThreadAllToAll(world)

    def rank_fn(r, _exchange):
        ops = CudaOps(scale)
        o, lse = ulysses_attention_forward(part(dq, r), part(dk, r), part(dv, r), scale, causal, ops=ops,
                                           alltoall=comm.make(r), rank=r, world=world)
        grads = ulysses_attention_backward(part(dq, r), part(dk, r), part(dv, r), o, lse, part(ddo, r), scale,
                                           causal, ops=ops, alltoall=comm.make(r), rank=r, world=world)
        return (o, lse) + grads

    res = _run_ranks_in_threads(world, rank_fn)
    assert fa.fa_check_status(torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    cat = [torch.cat([res[r][i] for r in range(world)], dim=2).cpu() for i in range(5)]
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, scale, causal, dtype)
    compare(cat[0], cat[1], o_ref, lse_ref, dtype)
    refs = oracle.attn_bwd(q, k, v, dout, scale, causal, dtype, magnitudes=True)
    print(compare_bwd(tuple(cat[2:]), refs[:3], refs[3:], dtype, q, k, dout, scale, causal))

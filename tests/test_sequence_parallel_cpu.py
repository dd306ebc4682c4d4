"""Multi-rank sequence-parallel attention on CPU: gloo ranks (spawned
processes) run the ring and all-gather schedules of
tiled_attention_18_b200.sequence_parallel with an fp64 oracle stand-in for the
kernels; the gathered result must equal full attention."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from tiled_attention_18_b200.sequence_parallel import (allgather_attention_forward, ring_attention_forward,
                                                       ring_schedule)


class OracleOps:
    """Partial attention by the fp64 oracle, fp64 LSE merge (test stand-in)."""

    def __init__(self, scale, dtype):
        self.scale, self.dtype = scale, dtype

    def partial(self, q, k, v, causal):
        import oracle
        o, lse = oracle.attn_fwd_gen(q, k, v, self.scale, causal, self.dtype)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def init(self, q):
        B, H, S, D = q.shape
        return [torch.zeros((B, H, S, D), dtype=torch.float64), torch.full((B, H, S), float("-inf"),
                                                                           dtype=torch.float64)]

    def merge(self, state, o_p, lse_p):
        o, lse = state
        m = torch.maximum(lse, lse_p)
        wa = torch.where(torch.isneginf(lse), torch.zeros_like(lse), torch.exp(lse - m))
        wb = torch.where(torch.isneginf(lse_p), torch.zeros_like(lse_p), torch.exp(lse_p - m))
        state[0] = (wa[..., None] * o + wb[..., None] * o_p) / (wa + wb)[..., None]
        state[1] = m + torch.log(wa + wb)

    def finalize(self, state):
        return state[0], state[1]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, mode, causal, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from tiled_attention_18_b200.workloads import make_inputs
        B, H, c, D = 1, 2, 24, 16
        q, k, v = make_inputs(B, H, world * c, D, "fp16", seed=5)
        sl = slice(rank * c, (rank + 1) * c)
        ops = OracleOps(0.25, "fp16")
        fn = ring_attention_forward if mode == "ring" else allgather_attention_forward
        o, lse = fn(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous(), 0.25, causal,
                    ops=ops)
        np.save(os.path.join(out_dir, f"o{rank}.npy"), o.numpy())
        np.save(os.path.join(out_dir, f"l{rank}.npy"), lse.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("mode", ["ring", "allgather"])
@pytest.mark.parametrize("causal", [False, True])
def test_sequence_parallel_ranks_equal_full_attention(tmp_path, world, mode, causal):
    import oracle
    from tiled_attention_18_b200.workloads import make_inputs
    mp.spawn(_worker, args=(world, _free_port(), mode, causal, str(tmp_path)), nprocs=world, join=True)
    B, H, c, D = 1, 2, 24, 16
    q, k, v = make_inputs(B, H, world * c, D, "fp16", seed=5)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, 0.25, causal, "fp16")
    o = np.concatenate([np.load(tmp_path / f"o{r}.npy") for r in range(world)], axis=2)
    lse = np.concatenate([np.load(tmp_path / f"l{r}.npy") for r in range(world)], axis=2)
    assert np.max(np.abs(o - o_ref)) <= 1e-12
    assert np.max(np.abs(lse - lse_ref)) <= 1e-12


def test_ring_schedule():
    assert ring_schedule(0, 3, False) == [(0, "full"), (2, "full"), (1, "full")]
    assert ring_schedule(2, 3, True) == [(2, "causal"), (1, "full"), (0, "full")]
    assert ring_schedule(0, 3, True) == [(0, "causal"), (2, "skip"), (1, "skip")]
    assert ring_schedule(1, 4, True) == [(1, "causal"), (0, "full"), (3, "skip"), (2, "skip")]


class GradOps:
    """Stand-in for the kernels in the ring backward: a block's share of the
    gradients for the rows' global O and LSE, in float64 (test stand-in)."""

    def __init__(self, scale):
        self.scale = scale

    def zeros_f32(self, t):
        return torch.zeros(t.shape, dtype=torch.float64)

    def bwd_partial(self, q, k, v, o, lse, dout, causal, deterministic=False):
        qd, kd, vd, dod = (t.double() for t in (q, k, v, dout))
        s = self.scale * qd @ kd.transpose(-1, -2)
        if causal:
            n = s.shape[-1]
            s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
        p = torch.exp(s - lse[..., None])
        ds = p * (dod @ vd.transpose(-1, -2) - (dod * o).sum(-1, keepdim=True))
        return self.scale * ds @ kd, self.scale * ds.transpose(-1, -2) @ qd, p.transpose(-1, -2) @ dod

    def accumulate(self, acc, x):
        acc += x

    def to16(self, acc, dtype):
        return acc


def _bwd_worker(rank, world, port, causal, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from tiled_attention_18_b200.sequence_parallel import ring_attention_backward
        from tiled_attention_18_b200.workloads import make_inputs
        B, H, c, D = 1, 2, 20, 16
        q, k, v = make_inputs(B, H, world * c, D, "bf16", seed=6)
        dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16)
        o, lse = oracle.attn_fwd(q, k, v, 0.25, causal, "bf16")  # the forward's global rows
        sl = slice(rank * c, (rank + 1) * c)
        part = lambda t: t[:, :, sl].contiguous()  # noqa: E731
        dq, dk, dv = ring_attention_backward(part(q), part(k), part(v), torch.from_numpy(o[:, :, sl].copy()),
                                             torch.from_numpy(lse[:, :, sl].copy()), part(dout), 0.25, causal,
                                             ops=GradOps(0.25))
        for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
            np.save(os.path.join(out_dir, f"{name}{rank}.npy"), t.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_backward_ranks_equal_full_gradients(tmp_path, world, causal):
    """The gradients gathered from the ranks equal the oracle's gradients of
    attention over the whole sequence."""
    import oracle
    from tiled_attention_18_b200.workloads import make_inputs
    mp.spawn(_bwd_worker, args=(world, _free_port(), causal, str(tmp_path)), nprocs=world, join=True)
    B, H, c, D = 1, 2, 20, 16
    q, k, v = make_inputs(B, H, world * c, D, "bf16", seed=6)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16)
    refs = oracle.attn_bwd(q, k, v, dout, 0.25, causal, "bf16")
    for name, ref in zip(("dq", "dk", "dv"), refs):
        got = np.concatenate([np.load(tmp_path / f"{name}{r}.npy") for r in range(world)], axis=2)
        assert np.max(np.abs(got - ref)) <= 1e-10, name


def _ulysses_worker(rank, world, port, causal, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from tiled_attention_18_b200.sequence_parallel import ulysses_attention_backward, ulysses_attention_forward
        from tiled_attention_18_b200.workloads import make_inputs
        B, H, c, D = 1, 2 * world, 16, 8
        q, k, v = make_inputs(B, H, world * c, D, "bf16", seed=8)
        dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
        sl = slice(rank * c, (rank + 1) * c)
        part = lambda t: t[:, :, sl].contiguous()  # noqa: E731
        o, lse = ulysses_attention_forward(part(q), part(k), part(v), 0.25, causal, ops=OracleOps(0.25, "bf16"))
        # the backward with the oracle's global rows as the forward output (float64 stand-in)
        o_full, lse_full = oracle.attn_fwd(q, k, v, 0.25, causal, "bf16")
        dq, dk, dv = ulysses_attention_backward(part(q), part(k), part(v),
                                                torch.from_numpy(o_full[:, :, sl].copy()),
                                                torch.from_numpy(lse_full[:, :, sl].copy()), part(dout), 0.25,
                                                causal, ops=GradOps(0.25))
        for name, t in (("o", o), ("l", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
            np.save(os.path.join(out_dir, f"u{name}{rank}.npy"), t.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ulysses_ranks_equal_full_attention(tmp_path, world, causal):
    """Head-parallel sequence parallelism over gloo: forward and backward equal
    the oracle over the whole sequence."""
    import oracle
    from tiled_attention_18_b200.workloads import make_inputs
    mp.spawn(_ulysses_worker, args=(world, _free_port(), causal, str(tmp_path)), nprocs=world, join=True)
    B, H, c, D = 1, 2 * world, 16, 8
    q, k, v = make_inputs(B, H, world * c, D, "bf16", seed=8)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, 0.25, causal, "bf16")
    refs = dict(zip(("dq", "dk", "dv"), oracle.attn_bwd(q, k, v, dout, 0.25, causal, "bf16")))
    refs.update(o=o_ref, l=lse_ref)
    for name, ref in refs.items():
        got = np.concatenate([np.load(tmp_path / f"u{name}{r}.npy") for r in range(world)], axis=2)
        assert np.max(np.abs(got - ref)) <= 1e-10, name


def test_single_rank_schedules_reduce_to_plain_attention():
    """World size 1 (no process group): every schedule is attention over the
    one chunk, forward and backward."""
    import oracle
    from tiled_attention_18_b200.sequence_parallel import (ring_attention_backward, ulysses_attention_backward,
                                                           ulysses_attention_forward)
    from tiled_attention_18_b200.workloads import make_inputs
    q, k, v = make_inputs(1, 2, 40, 8, "bf16", seed=21)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(22)).to(torch.bfloat16)
    for causal in (False, True):
        o_ref, lse_ref = oracle.attn_fwd(q, k, v, 0.25, causal, "bf16")
        ident = lambda x: x.clone()  # noqa: E731  (the one-rank all-to-all)
        outs = [ring_attention_forward(q, k, v, 0.25, causal, ops=OracleOps(0.25, "bf16"), rank=0, world=1),
                allgather_attention_forward(q, k, v, 0.25, causal, ops=OracleOps(0.25, "bf16"), rank=0, world=1,
                                            gather=lambda kv: kv[None]),
                ulysses_attention_forward(q, k, v, 0.25, causal, ops=OracleOps(0.25, "bf16"), alltoall=ident,
                                          rank=0, world=1)]
        for o, lse in outs:
            assert np.max(np.abs(o.numpy() - o_ref)) <= 1e-12
            assert np.max(np.abs(lse.numpy() - lse_ref)) <= 1e-12
        refs = oracle.attn_bwd(q, k, v, dout, 0.25, causal, "bf16")
        o64, l64 = torch.from_numpy(o_ref), torch.from_numpy(lse_ref)
        grads = [ring_attention_backward(q, k, v, o64, l64, dout, 0.25, causal, ops=GradOps(0.25), rank=0, world=1,
                                         exchange=lambda s, payload: (None, payload)),
                 ulysses_attention_backward(q, k, v, o64, l64, dout, 0.25, causal, ops=GradOps(0.25), alltoall=ident,
                                            rank=0, world=1)]
        for g in grads:
            for a, b in zip(g, refs):
                assert np.max(np.abs(a.numpy() - b)) <= 1e-10

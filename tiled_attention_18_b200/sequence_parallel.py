"""Sequence-parallel attention forward across the ranks of a torch.distributed group.

The sequence is split into equal contiguous chunks, one per rank in rank
order; every rank holds its chunk of Q, K and V ([B, H, c, D]) and computes
the attention of its queries over the whole sequence, the K/V it lacks coming
from the other ranks ("FlashAttention-2 在昇腾 NPU 上如何做到 3 倍加速？",
section 6.4: each device computes the attention of its part of the sequence,
K/V synchronised between devices by collective communication).  Two ways:

- ``allgather_attention_forward``: one all-gather of K and V, then one
  ``fa_fwd_ex`` over the keys this rank's queries can see (all of them, or,
  with the causal mask, the first (rank + 1) * c: bottom-right alignment puts
  query i of the chunk at global position rank * c + i).  Memory: the whole
  sequence's K/V on every rank.
- ``ring_attention_forward``: the K/V blocks travel around the ring (P2P to
  rank + 1, from rank - 1) while each rank computes the attention of its
  queries over the block it holds and folds the partial (O, LSE) into a
  running fp32 result with ``fa_merge_partial`` (the log-sum-exp merge).
  With the causal mask a rank skips the blocks that come after its own and
  uses the causal kernel on its own block.  Memory: two K/V blocks.

- ``ulysses_attention_forward`` / ``ulysses_attention_backward``: head
  parallelism inside the sequence-parallel group: one all-to-all gives each
  rank H / world heads over the whole sequence, the unmodified kernels run on
  them, and one all-to-all returns the results (no merge).

``ring_attention_backward`` gives the gradients of the ring forward (the
section's setting is distributed training): with the global O and LSE of the
forward, ``fa_bwd`` on (this rank's queries, one K/V block) yields exactly that
block's share of dQ, dK and dV, so dQ accumulates locally while every K/V
block travels the ring together with fp32 accumulators of its dK and dV
(``fa_accumulate``), one more step than the forward, back to its owner.

Every step of the attention runs in the library's kernels; this module only
orders the launches and the communication.  The ``ops`` and ``exchange``
parameters exist so that tests can drive the same schedule with stand-ins
(CPU ranks over gloo, or all ranks in one process on one GPU).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Tuple


def ring_schedule(rank: int, world: int, causal: bool) -> List[Tuple[int, str]]:
    """(source rank, mode) for ring steps s = 0 .. world - 1: at step s this rank
    holds the K/V block of rank (rank - s) mod world; mode is "full", "causal"
    (its own block under the mask) or "skip" (a block after its own under the
    mask)."""
    out = []
    for s in range(world):
        src = (rank - s) % world
        if not causal:
            out.append((src, "full"))
        elif src == rank:
            out.append((src, "causal"))
        elif src < rank:
            out.append((src, "full"))
        else:
            out.append((src, "skip"))
    return out


class CudaOps:
    """The library's kernels: fa_fwd_ex for a partial, fa_merge_partial /
    fa_merge_finalize for the running result (fp32 O, fp32 LSE)."""

    def __init__(self, scale: float, stream=None):
        self.scale = float(scale)
        self.stream = stream

    def _sid(self, t):
        import torch
        st = self.stream if self.stream is not None else torch.cuda.current_stream(t.device)
        return int(st.cuda_stream)

    def partial(self, q, k, v, causal: bool):
        from . import flash_attention_forward
        return flash_attention_forward(q, k, v, self.scale, causal, stream=self.stream)

    def init(self, q):
        import torch
        B, H, S, D = q.shape
        o = torch.zeros((B, H, S, D), dtype=torch.float32, device=q.device)
        lse = torch.full((B, H, S), float("-inf"), dtype=torch.float32, device=q.device)
        return [o, lse, q.dtype]

    def merge(self, state, o_part, lse_part):
        from . import FaError, fa_merge_partial
        from . import _dtype_code
        o_acc, lse_acc, _ = state
        rows = lse_acc.numel()
        rc = fa_merge_partial(o_acc.data_ptr(), lse_acc.data_ptr(), o_part.data_ptr(), lse_part.data_ptr(), rows,
                              o_acc.shape[-1], _dtype_code(o_part), self._sid(o_acc))
        if rc != 0:
            raise FaError(rc, "fa_merge_partial")

    # -- backward
    def __init_bwd(self, q):
        import torch
        from . import fa_bwd_workspace_size
        B, H, S, D = q.shape
        n = fa_bwd_workspace_size(B, H, S, D)
        if getattr(self, "_ws", None) is None or self._ws.numel() < n:
            self._ws = torch.empty(max(n, 1), dtype=torch.uint8, device=q.device)

    def zeros_f32(self, t):
        import torch
        return torch.zeros(t.shape, dtype=torch.float32, device=t.device)

    def bwd_partial(self, q, k, v, o, lse, dout, causal: bool, deterministic: bool = False):
        """This block's share of dQ, dK, dV (16-bit) for the rows' global O and LSE."""
        from . import flash_attention_backward
        self.__init_bwd(q)
        return flash_attention_backward(q, k.contiguous(), v.contiguous(), o, lse, dout, self.scale, causal,
                                        deterministic=deterministic, workspace=self._ws, stream=self.stream)

    def accumulate(self, acc, x):
        from . import FaError, fa_accumulate
        code = 1 if str(x.dtype) == "torch.bfloat16" else 0
        rc = fa_accumulate(acc.data_ptr(), x.data_ptr(), x.numel(), code, self._sid(acc))
        if rc != 0:
            raise FaError(rc, "fa_accumulate")

    def to16(self, acc, dtype):
        import torch
        from . import FaError, fa_merge_finalize
        out = torch.empty(acc.shape, dtype=dtype, device=acc.device)
        code = 1 if dtype == torch.bfloat16 else 0
        rc = fa_merge_finalize(acc.data_ptr(), out.data_ptr(), acc.numel(), code, self._sid(acc))
        if rc != 0:
            raise FaError(rc, "fa_merge_finalize")
        return out

    def finalize(self, state):
        import torch
        from . import FaError, fa_merge_finalize
        o_acc, lse_acc, dtype = state
        o = torch.empty(o_acc.shape, dtype=dtype, device=o_acc.device)
        code = 1 if dtype == torch.bfloat16 else 0
        rc = fa_merge_finalize(o_acc.data_ptr(), o.data_ptr(), o_acc.numel(), code, self._sid(o_acc))
        if rc != 0:
            raise FaError(rc, "fa_merge_finalize")
        return o, lse_acc


def _p2p_ring_exchange(group, rank: int, world: int):
    """Send the held K/V block to rank + 1 and receive the next from rank - 1
    (one packed buffer per step)."""
    import torch
    import torch.distributed as dist

    nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world

    def exchange(step: int, kv):
        recv = torch.empty_like(kv)
        ops = [dist.P2POp(dist.isend, kv, nxt, group), dist.P2POp(dist.irecv, recv, prv, group)]
        reqs = dist.batch_isend_irecv(ops)
        return reqs, recv

    return exchange


def ring_attention_forward(q, k, v, scale: float, causal: bool = False, group=None, ops=None,
                           exchange: Optional[Callable] = None, rank: Optional[int] = None,
                           world: Optional[int] = None):
    """O and LSE of this rank's query chunk over the whole sequence.

    q, k, v: this rank's contiguous chunks [B, H, c, D] (equal c on every rank).
    With the default ``exchange`` the K/V blocks move by NCCL (or gloo) P2P on
    ``group``; the transfer of step s + 1's block is started before step s's
    attention and waited for after it, so the two overlap.
    """
    import torch
    import torch.distributed as dist

    if rank is None:
        rank = dist.get_rank(group)
    if world is None:
        world = dist.get_world_size(group)
    ops = ops if ops is not None else CudaOps(scale)
    if exchange is None:
        exchange = _p2p_ring_exchange(group, rank, world)
    c = k.shape[2]
    kv = torch.stack([k, v])  # one buffer per step: [2, B, H, c, D]
    state = ops.init(q)
    for s, (src, mode) in enumerate(ring_schedule(rank, world, causal)):
        pending = exchange(s, kv) if s + 1 < world else None
        if mode != "skip":
            o_p, lse_p = ops.partial(q, kv[0], kv[1], mode == "causal")
            ops.merge(state, o_p, lse_p)
        if pending is not None:
            reqs, nxt = pending
            for r in reqs or []:
                r.wait()
            kv = nxt
    assert kv.shape[3] == c
    return ops.finalize(state)


def allgather_attention_forward(q, k, v, scale: float, causal: bool = False, group=None, ops=None,
                                gather: Optional[Callable] = None, rank: Optional[int] = None,
                                world: Optional[int] = None):
    """O and LSE of this rank's query chunk: all-gather K and V, then one
    partial over the visible keys (all of them, or the first (rank + 1) * c
    with the causal mask, aligned bottom-right)."""
    import torch
    import torch.distributed as dist

    if rank is None:
        rank = dist.get_rank(group)
    if world is None:
        world = dist.get_world_size(group)
    ops = ops if ops is not None else CudaOps(scale)
    B, H, c, D = k.shape
    kv = torch.stack([k, v]).contiguous()
    if gather is None:
        # the concatenated form [world * 2, ...] (every backend accepts it)
        out = torch.empty((world * 2,) + tuple(kv.shape[1:]), dtype=kv.dtype, device=kv.device)
        dist.all_gather_into_tensor(out, kv, group=group)
        out = out.view((world,) + tuple(kv.shape))
    else:
        out = gather(kv)
    # [world, 2, B, H, c, D] -> K, V [B, H, world * c, D] (rank-ordered chunks)
    full = out.permute(1, 2, 3, 0, 4, 5).reshape(2, B, H, world * c, D)
    n_keys = (rank + 1) * c if causal else world * c
    kf = full[0, :, :, :n_keys].contiguous()
    vf = full[1, :, :, :n_keys].contiguous()
    return ops.partial(q, kf, vf, causal)


def _p2p_ring_exchange_tuple(group, rank: int, world: int):
    """Send a tuple of tensors to rank + 1 and receive tensors of the same shapes
    from rank - 1 (one batched P2P call per step)."""
    import torch
    import torch.distributed as dist

    nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world

    def exchange(step: int, payload):
        recv = tuple(torch.empty_like(t) for t in payload)
        ops = [dist.P2POp(dist.isend, t, nxt, group) for t in payload]
        ops += [dist.P2POp(dist.irecv, r, prv, group) for r in recv]
        return dist.batch_isend_irecv(ops), recv

    return exchange


def ring_attention_backward(q, k, v, o, lse, dout, scale: float, causal: bool = False, group=None, ops=None,
                            exchange: Optional[Callable] = None, rank: Optional[int] = None,
                            world: Optional[int] = None, deterministic: bool = False):
    """dQ, dK, dV of this rank's chunks for the ring forward.

    q, k, v, dout: this rank's chunks [B, H, c, D]; o, lse: this rank's rows of
    the forward over the whole sequence (ring_attention_forward's output).  At
    step s the rank holds the K/V block of rank (rank - s) mod world with the
    fp32 dK/dV accumulated for it so far, adds its queries' share, and passes
    both on; after world exchanges each rank holds its own block again with
    every rank's share added.  dQ is summed locally in fp32.  The causal mask
    skips blocks after the rank's own and uses the causal kernel on its own.
    """
    import torch
    import torch.distributed as dist

    if rank is None:
        rank = dist.get_rank(group)
    if world is None:
        world = dist.get_world_size(group)
    ops = ops if ops is not None else CudaOps(scale)
    if exchange is None:
        exchange = _p2p_ring_exchange_tuple(group, rank, world)
    kv = torch.stack([k, v])                 # the block being carried: [2, B, H, c, D]
    acc = ops.zeros_f32(kv)                  # its dK, dV so far (fp32)
    dq_acc = ops.zeros_f32(q)
    for s, (src, mode) in enumerate(ring_schedule(rank, world, causal)):
        if mode != "skip":
            dq_p, dk_p, dv_p = ops.bwd_partial(q, kv[0], kv[1], o, lse, dout, mode == "causal", deterministic)
            ops.accumulate(dq_acc, dq_p)
            ops.accumulate(acc[0], dk_p)
            ops.accumulate(acc[1], dv_p)
        reqs, (kv, acc) = exchange(s, (kv, acc))
        for r in reqs or []:
            r.wait()
    return ops.to16(dq_acc, q.dtype), ops.to16(acc[0], k.dtype), ops.to16(acc[1], v.dtype)


# ------------------------------------------------------------------ all-to-all (head-parallel)

def _alltoall_default(group, world: int):
    """all_to_all over ``group`` of a tensor whose leading dimension indexes the
    destination rank; returns the tensor whose leading dimension indexes the source."""
    import torch
    import torch.distributed as dist

    def a2a(x):
        out = torch.empty_like(x)
        dist.all_to_all_single(out, x.contiguous(), group=group)
        return out

    return a2a


def _to_heads(x, world: int, c: int):
    """[B, H, c, D] chunk (this rank's positions, all heads) -> [world, B, H/world, c, D],
    leading dimension = the rank that owns that head group."""
    B, H, _, D = x.shape
    return x.reshape(B, world, H // world, c, D).permute(1, 0, 2, 3, 4)


def _gather_positions(y, world: int, c: int):
    """[world(source), B, Hw, c, D] -> [B, Hw, world * c, D]: the source ranks' chunks in
    sequence order."""
    W, B, Hw, _, D = y.shape
    return y.permute(1, 2, 0, 3, 4).reshape(B, Hw, W * c, D)


def _scatter_positions(x, world: int, c: int):
    """[B, Hw, world * c, ...] -> [world(destination), B, Hw, c, ...]."""
    B, Hw = x.shape[:2]
    rest = tuple(x.shape[3:])
    return x.reshape((B, Hw, world, c) + rest).permute((2, 0, 1, 3) + tuple(range(4, 4 + len(rest))))


def _back_to_chunk(y, world: int):
    """[world(source = head group), B, Hw, c, ...] -> [B, world * Hw, c, ...] (all heads
    of this rank's positions)."""
    W, B, Hw, c = y.shape[:4]
    rest = tuple(y.shape[4:])
    return y.permute((1, 0, 2, 3) + tuple(range(4, 4 + len(rest)))).reshape((B, W * Hw, c) + rest)


def ulysses_attention_forward(q, k, v, scale: float, causal: bool = False, group=None, ops=None,
                              alltoall: Optional[Callable] = None, rank: Optional[int] = None,
                              world: Optional[int] = None):
    """O and LSE of this rank's query chunk by head-parallel attention: one
    all-to-all turns the sequence-sharded Q, K, V ([B, H, c, D] per rank) into
    head-sharded full sequences ([B, H / world, world * c, D]), each rank runs
    the attention of its heads over the whole sequence (causal mask included,
    the positions being in order), and one all-to-all returns O and LSE to the
    ranks that own the positions.  H must be a multiple of world.  No merge is
    needed: each head's attention runs in one kernel call."""
    import torch
    import torch.distributed as dist

    if rank is None:
        rank = dist.get_rank(group)
    if world is None:
        world = dist.get_world_size(group)
    B, H, c, D = q.shape
    if H % world:
        raise ValueError("the head count must be a multiple of the group size")
    ops = ops if ops is not None else CudaOps(scale)
    a2a = alltoall if alltoall is not None else _alltoall_default(group, world)
    recv = a2a(torch.stack([_to_heads(t, world, c) for t in (q, k, v)], dim=1))  # [W, 3, B, Hw, c, D]
    qh, kh, vh = (_gather_positions(recv[:, i], world, c).contiguous() for i in range(3))
    o, lse = ops.partial(qh, kh, vh, causal)
    o_back = a2a(_scatter_positions(o, world, c).contiguous())             # [W, B, Hw, c, D]
    l_back = a2a(_scatter_positions(lse, world, c).contiguous())           # [W, B, Hw, c]
    return _back_to_chunk(o_back, world).contiguous(), _back_to_chunk(l_back, world).contiguous()


def ulysses_attention_backward(q, k, v, o, lse, dout, scale: float, causal: bool = False, group=None, ops=None,
                               alltoall: Optional[Callable] = None, rank: Optional[int] = None,
                               world: Optional[int] = None, deterministic: bool = False):
    """dQ, dK, dV of this rank's chunks for ulysses_attention_forward: the
    inputs, O, dO and LSE go to the head owners by one all-to-all, each rank
    runs the backward of its heads over the whole sequence, and the gradients
    come back by another."""
    import torch
    import torch.distributed as dist

    if rank is None:
        rank = dist.get_rank(group)
    if world is None:
        world = dist.get_world_size(group)
    B, H, c, D = q.shape
    ops = ops if ops is not None else CudaOps(scale)
    a2a = alltoall if alltoall is not None else _alltoall_default(group, world)
    recv = a2a(torch.stack([_to_heads(t, world, c) for t in (q, k, v, o, dout)], dim=1))  # [W, 5, B, Hw, c, D]
    qh, kh, vh, oh, doh = (_gather_positions(recv[:, i], world, c).contiguous() for i in range(5))
    lh = a2a(lse.reshape(B, world, H // world, c).permute(1, 0, 2, 3).contiguous())      # [W, B, Hw, c]
    lh = lh.permute(1, 2, 0, 3).reshape(B, H // world, world * c).contiguous()
    dq, dk, dv = ops.bwd_partial(qh, kh, vh, oh, lh, doh, causal, deterministic)
    grads = a2a(torch.stack([_scatter_positions(g, world, c) for g in (dq, dk, dv)], dim=1).contiguous())
    return tuple(_back_to_chunk(grads[:, i], world).contiguous() for i in range(3))

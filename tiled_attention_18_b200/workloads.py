"""Seeded synthetic inputs for the attention forward pass.

This module holds the workload definitions and the input generator that both
the CUDA path's tests/benchmark and the fp64 oracle read.  It contains none of
the method's arithmetic: it draws Gaussian samples and rounds them to the
16-bit input dtype, nothing else.

Recipe (every workload): one ``torch.Generator`` on the CPU seeded with the
workload's seed (0 unless stated), ``randn`` in float32 drawn in the order
Q, K, V with shape [B, H, S, D]; Q and K are multiplied by ``qk_mult`` (an
exact power of two) in float32; then all three are rounded to the dtype
(round-to-nearest-even, torch's conversion) and made contiguous (BHSD).
The same 16-bit values are copied to the GPU and handed to the oracle.

The shapes follow the pages' workloads: the ops-transformer page's
B=2, H=12, S=2048, D=64 causal run ("ops-transformer FlashAttention 算子实战"
section 4.1-4.2); a 13B-style decoder layer at S=8192 (the gsyq.cn catlass
page's 13B service, BF16 above 4K); the learning-hub tutorial's
B=1, H=32, S=2048, D=128 fp16 check; and long-context S=16384 runs.  Gaussian
activations stand in for the models' activations (no weights are used).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    S: int
    D: int
    dtype: str          # "fp16" | "bf16"
    causal: bool
    qk_mult: float = 1.0
    seed: int = 0
    Sk: int = 0            # keys per head; 0 = S (self-attention)
    layout: str = "bhsd"   # memory layout of Q, K, V and O: "bhsd" or "bshd"

    @property
    def Skv(self) -> int:
        return self.Sk if self.Sk else self.S

    @property
    def general(self) -> bool:
        """True when the workload needs fa_fwd_ex (Sq != Sk or a non-BHSD layout)."""
        return self.Skv != self.S or self.layout != "bhsd"

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float16 if self.dtype == "fp16" else torch.bfloat16

    @property
    def scale(self) -> float:
        return softmax_scale(self.D)

    @property
    def flops(self) -> float:
        if not self.general:
            return attention_flops(self.B, self.H, self.S, self.D, self.causal)
        return attention_flops_general(self.B, self.H, self.S, self.Skv, self.D, self.causal)

    def describe(self) -> str:
        c = "causal" if self.causal else "non-causal"
        extra = f", Q,K x{self.qk_mult:g}" if self.qk_mult != 1.0 else ""
        if self.general:
            lay = f", {self.layout.upper()}" if self.layout != "bhsd" else ""
            return (f"attn-fwd {self.dtype} B={self.B} H={self.H} Sq={self.S} Sk={self.Skv} D={self.D} "
                    f"{c}{extra}{lay}")
        return f"attn-fwd {self.dtype} B={self.B} H={self.H} S={self.S} D={self.D} {c}{extra}"


def softmax_scale(D: int) -> float:
    """The caller's scale 1/sqrt(D), computed in float32 (as a float32 value)."""
    return float(np.float32(1.0) / np.sqrt(np.float32(D)))


def attention_flops(B: int, H: int, S: int, D: int, causal: bool) -> float:
    """Algorithmic FLOPs of the two matmuls, 4*B*H*S^2*D, halved when causal."""
    f = 4.0 * B * H * S * S * D
    return f / 2.0 if causal else f


def attention_flops_general(B: int, H: int, Sq: int, Sk: int, D: int, causal: bool) -> float:
    """4*B*H*Sq*Sk*D; with the bottom-right causal mask the Sq x Sq corner above
    the diagonal is not counted (half of it), which gives attention_flops when
    Sq = Sk."""
    f = 4.0 * B * H * Sq * Sk * D
    if causal:
        f -= 4.0 * B * H * D * Sq * Sq / 2.0
    return f


# The five workload configurations; the last one runs both with and without the mask.
WORKLOADS = {
    "c1": Workload("c1", 1, 2, 256, 64, "fp16", False),
    "c2": Workload("c2", 1, 32, 2048, 128, "fp16", False),
    "c3": Workload("c3", 2, 12, 2048, 64, "fp16", True),
    "c4": Workload("c4", 1, 40, 8192, 128, "bf16", True, qk_mult=2.0),
    "c5a": Workload("c5a", 1, 32, 16384, 128, "bf16", False),
    "c5b": Workload("c5b", 1, 32, 16384, 128, "bf16", True),
}

# General-shape workloads (fa_fwd_ex):
# - sdxl_xattn: text-to-image cross-attention, 4096 image tokens (a 64 x 64
#   latent grid) attending to 77 text tokens, 10 heads of 64 (the SDXL case of
#   "解析CANN ops-transformer的FlashAttention算子：注意力机制的内存优化");
# - bert_large: the BERT-Large shape B=32, H=16, S=512, D=64 of the
#   FlashAttention-2 page's section 4.3, with the tensors in the
#   [batch, seq_len, heads, head_dim] layout that the gsyq.cn catlass page warns
#   about, read in place;
# - prefill_cached: a causal chunk of 4096 new queries over 16384 cached keys
#   (queries aligned to the last keys), bf16 as the catlass page advises above 4K;
# - d256_long: head dimension 256, S = 8192, causal, bf16.
GENERAL_WORKLOADS = {
    "sdxl_xattn": Workload("sdxl_xattn", 2, 10, 4096, 64, "fp16", False, Sk=77),
    "bert_large": Workload("bert_large", 32, 16, 512, 64, "fp16", False, layout="bshd"),
    "prefill_cached": Workload("prefill_cached", 1, 32, 4096, 128, "bf16", True, Sk=16384),
    # head dimension 256 (the third of the pages' common head dimensions), long context
    "d256_long": Workload("d256_long", 1, 16, 8192, 256, "bf16", True),
}

# Parity tolerances (max-abs) on O by dtype, and on the LSE.
O_TOL = {"fp16": 2e-3, "bf16": 1e-2}
LSE_TOL = 1e-3


def make_inputs(B: int, H: int, S: int, D: int, dtype: str, qk_mult: float = 1.0, seed: int = 0):
    """Q, K, V as contiguous CPU tensors of the 16-bit dtype (see module doc)."""
    tdt = torch.float16 if dtype == "fp16" else torch.bfloat16
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    shape = (B, H, S, D)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    if qk_mult != 1.0:
        assert math.log2(qk_mult).is_integer(), "qk_mult must be a power of two"
        q.mul_(qk_mult)
        k.mul_(qk_mult)
    return (q.to(tdt).contiguous(), k.to(tdt).contiguous(), v.to(tdt).contiguous())


def make_cross_inputs(B: int, H: int, Sq: int, Sk: int, D: int, dtype: str, seed: int = 0):
    """Q [B,H,Sq,D] drawn as make_inputs(seed) draws Q; K, V [B,H,Sk,D] drawn as
    make_inputs(seed + 1) draws K and V.  Contiguous BHSD CPU tensors."""
    q, _, _ = make_inputs(B, H, Sq, D, dtype, seed=seed)
    _, k, v = make_inputs(B, H, Sk, D, dtype, seed=seed + 1)
    return q, k, v


def to_layout(x: torch.Tensor, layout: str) -> torch.Tensor:
    """The same [B,H,S,D] values stored in ``layout``, returned as a [B,H,S,D] view."""
    if layout == "bhsd":
        return x.contiguous()
    if layout == "bshd":
        return x.transpose(1, 2).contiguous().transpose(1, 2)
    raise ValueError(f"unknown layout {layout!r}")


def workload_inputs(w: Workload):
    """Contiguous BHSD CPU tensors of the workload (see to_layout for its layout)."""
    if w.Skv != w.S:
        return make_cross_inputs(w.B, w.H, w.S, w.Skv, w.D, w.dtype, w.seed)
    return make_inputs(w.B, w.H, w.S, w.D, w.dtype, w.qk_mult, w.seed)


def sample_rows(B: int, H: int, S: int, n_random: int, edge: int = 2, seed: int = 1234):
    """Row sample for full-size checks: for every (b,h) the first and last ``edge``
    rows, plus ``n_random`` seeded random (bh, row) pairs; sorted by bh."""
    rng = np.random.default_rng(seed)
    bh_list, row_list = [], []
    for bh in range(B * H):
        rows = list(range(min(edge, S))) + list(range(max(S - edge, 0), S))
        bh_list += [bh] * len(rows)
        row_list += rows
    bh_list += list(rng.integers(0, B * H, size=n_random))
    row_list += list(rng.integers(0, S, size=n_random))
    bh_arr = np.asarray(bh_list, dtype=np.int64)
    row_arr = np.asarray(row_list, dtype=np.int64)
    order = np.lexsort((row_arr, bh_arr))
    return bh_arr[order], row_arr[order]

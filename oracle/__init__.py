"""fp64 CPU oracle for the attention forward pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library in
``tiled_attention_18_b200`` and its binding) never imports, links or calls it.
It shares no code with the CUDA path; the two meet only in the seeded input
generators of ``tiled_attention_18_b200.workloads``, which hold none of the
method's arithmetic.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, OpenMP over rows);
this module builds it with gcc when needed and marshals numpy arrays through
ctypes.  Function-level citations are in the C file's header:
- ``attn_fwd``   : the definition softmax(scale * Q K^T [+ causal]) V and the
  per-row log-sum-exp ("FlashAttention-2 在昇腾 NPU 上如何做到 3 倍加速？" section 1;
  "ops-transformer FlashAttention 算子实战" section 4.2).
- ``attn_rows``  : the same definition for sampled rows.
- ``attn_tiled`` : the tiled online-softmax recurrence of the FlashAttention-2
  page, sections 2.1-2.2, with causal key-tile skipping (gsyq.cn catlass
  page, "Causal Mask的实现差异", mode 2).
- ``attn_probs`` : the softmax matrix P of one head (tiny sizes).
- ``causal_tile_count`` : element-wise enumeration of computed/skipped tile pairs.
- ``attn_fwd_gen`` / ``attn_rows_gen`` : the same definition with Sq queries and
  Sk keys (cross-attention) and the causal mask aligned to the last Sq keys.
- ``attn_bwd`` : dQ, dK, dV by the chain rule through the definition (the
  softmax Jacobian), with optional absolute-value error scales.
- ``attn_fwd_masked`` / ``attn_bwd_masked`` : the definition with an explicit
  boolean mask, and its gradients.
- ``philox4x32_10`` / ``dropout_keep_mask`` : the counter-based generator
  (Salmon et al., SC 2011) and the keep decisions of attention dropout.
- ``attn_fwd_dropout`` / ``attn_rows_dropout`` / ``attn_bwd_dropout`` :
  attention with dropout after the softmax (FlashAttention-2 page, sections
  3.4 and 6.3) and its gradients.

Parity pins: every function above is pinned by tests in tests/test_oracle.py and
tests/test_oracle_general.py (torch SDPA in float64 with an explicit mask, the
Q = 0 closed form, agreement with attn_fwd when Sq = Sk) and
tests/test_oracle_bwd.py (float64 autograd, central finite differences of
attn_fwd_gen, closed forms and column-sum identities) and
tests/test_oracle_mask.py (SDPA fp64 with a boolean mask, all-ones mask =
no mask, lower-triangular mask = the causal flag, fully masked rows) and
tests/test_oracle_dropout.py (Philox known-answer vectors, keep rates, p = 0
equals no dropout, unbiasedness over offsets, float64 autograd).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F16 = 0
BF16 = 1


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        u16p = ctypes.POINTER(ctypes.c_uint16)
        f64p = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_f64.restype = ctypes.c_double
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_decode.argtypes = [u16p, f64p, i64, ctypes.c_int]
        lib.oracle_decode.restype = None
        lib.oracle_attn_fwd.argtypes = [u16p, u16p, u16p, i64, i64, i64, i64, ctypes.c_float,
                                        ctypes.c_int, ctypes.c_int, f64p, f64p]
        lib.oracle_attn_fwd.restype = ctypes.c_int
        lib.oracle_attn_rows.argtypes = [u16p, u16p, u16p, i64, i64, i64, i64, ctypes.c_float,
                                         ctypes.c_int, ctypes.c_int, i64p, i64p, i64, f64p, f64p]
        lib.oracle_attn_rows.restype = ctypes.c_int
        lib.oracle_attn_probs.argtypes = [u16p, u16p, i64, i64, i64, i64, ctypes.c_float,
                                          ctypes.c_int, ctypes.c_int, i64, f64p]
        lib.oracle_attn_probs.restype = ctypes.c_int
        lib.oracle_attn_tiled.argtypes = [u16p, u16p, u16p, i64, i64, i64, i64, ctypes.c_float,
                                          ctypes.c_int, ctypes.c_int, i64, i64, ctypes.c_int,
                                          f64p, f64p]
        lib.oracle_attn_tiled.restype = ctypes.c_int
        lib.oracle_attn_fwd_gen.argtypes = [u16p, u16p, u16p, i64, i64, i64, i64, i64, ctypes.c_float,
                                            ctypes.c_int, ctypes.c_int, f64p, f64p]
        lib.oracle_attn_fwd_gen.restype = ctypes.c_int
        lib.oracle_attn_rows_gen.argtypes = [u16p, u16p, u16p, i64, i64, i64, i64, i64, ctypes.c_float,
                                             ctypes.c_int, ctypes.c_int, i64p, i64p, i64, f64p, f64p]
        lib.oracle_attn_rows_gen.restype = ctypes.c_int
        lib.oracle_attn_bwd.argtypes = [u16p, u16p, u16p, u16p, i64, i64, i64, i64, i64, ctypes.c_float,
                                        ctypes.c_int, ctypes.c_int, f64p, f64p, f64p, f64p, f64p, f64p]
        lib.oracle_attn_bwd.restype = ctypes.c_int
        lib.oracle_attn_fwd_masked.argtypes = [u16p, u16p, u16p, i64, i64, i64, i64, i64, ctypes.c_float,
                                               ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_uint8), i64, i64,
                                               i64, f64p, f64p]
        lib.oracle_attn_fwd_masked.restype = ctypes.c_int
        lib.oracle_attn_bwd_masked.argtypes = [u16p, u16p, u16p, u16p, i64, i64, i64, i64, i64, ctypes.c_float,
                                               ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_uint8), i64, i64,
                                               i64, f64p, f64p, f64p, f64p, f64p, f64p]
        lib.oracle_attn_bwd_masked.restype = ctypes.c_int
        u32 = ctypes.c_uint32
        u32p = ctypes.POINTER(ctypes.c_uint32)
        lib.oracle_philox4x32_10.argtypes = [u32p, u32p, u32p]
        lib.oracle_philox4x32_10.restype = None
        lib.oracle_dropout_keep_mask.argtypes = [i64, i64, i64, u32, ctypes.c_uint64, u32,
                                                 ctypes.POINTER(ctypes.c_uint8)]
        lib.oracle_dropout_keep_mask.restype = ctypes.c_int
        lib.oracle_attn_fwd_dropout.argtypes = [u16p, u16p, u16p, i64, i64, i64, i64, i64, ctypes.c_float,
                                                ctypes.c_int, ctypes.c_int, u32, ctypes.c_uint64, u32, f64p, f64p]
        lib.oracle_attn_fwd_dropout.restype = ctypes.c_int
        u8p = ctypes.POINTER(ctypes.c_uint8)
        lib.oracle_attn_fwd_dropout_masked.argtypes = [u16p, u16p, u16p, i64, i64, i64, i64, i64, ctypes.c_float,
                                                       ctypes.c_int, ctypes.c_int, u32, ctypes.c_uint64, u32, u8p,
                                                       i64, i64, i64, f64p, f64p]
        lib.oracle_attn_fwd_dropout_masked.restype = ctypes.c_int
        lib.oracle_attn_bwd_dropout_masked.argtypes = [u16p, u16p, u16p, u16p, i64, i64, i64, i64, i64,
                                                       ctypes.c_float, ctypes.c_int, ctypes.c_int, u32,
                                                       ctypes.c_uint64, u32, u8p, i64, i64, i64, f64p, f64p, f64p,
                                                       f64p, f64p, f64p]
        lib.oracle_attn_bwd_dropout_masked.restype = ctypes.c_int
        lib.oracle_attn_rows_dropout.argtypes = [u16p, u16p, u16p, i64, i64, i64, i64, i64, ctypes.c_float,
                                                 ctypes.c_int, ctypes.c_int, u32, ctypes.c_uint64, u32, i64p, i64p,
                                                 i64, f64p, f64p]
        lib.oracle_attn_rows_dropout.restype = ctypes.c_int
        lib.oracle_attn_bwd_dropout.argtypes = [u16p, u16p, u16p, u16p, i64, i64, i64, i64, i64, ctypes.c_float,
                                                ctypes.c_int, ctypes.c_int, u32, ctypes.c_uint64, u32, f64p, f64p,
                                                f64p, f64p, f64p, f64p]
        lib.oracle_attn_bwd_dropout.restype = ctypes.c_int
        lib.oracle_causal_tile_count.argtypes = [i64, i64, i64, i64p, i64p, i64p]
        lib.oracle_causal_tile_count.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
        return lib


def _dtype_code(dtype) -> int:
    name = str(dtype).replace("torch.", "")
    if name in ("fp16", "float16", "half"):
        return F16
    if name in ("bf16", "bfloat16"):
        return BF16
    raise ValueError(f"oracle: unsupported dtype {dtype!r}")


def _bits(x) -> np.ndarray:
    """16-bit bit patterns of a torch fp16/bf16 tensor or a uint16 numpy array."""
    if isinstance(x, np.ndarray):
        if x.dtype == np.uint16:
            return np.ascontiguousarray(x)
        if x.dtype == np.float16:
            return np.ascontiguousarray(x).view(np.uint16)
        raise TypeError("oracle: numpy input must be uint16 bit patterns or float16")
    import torch  # local: only tensors need it
    t = x.detach().to("cpu").contiguous()
    if t.dtype not in (torch.float16, torch.bfloat16):
        raise TypeError("oracle: tensor input must be float16 or bfloat16")
    return t.view(torch.int16).numpy().view(np.uint16)


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def decode(bits: np.ndarray, dtype) -> np.ndarray:
    lib = _load()
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(b.shape, dtype=np.float64)
    lib.oracle_decode(_ptr(b, ctypes.c_uint16), _ptr(out, ctypes.c_double), b.size, _dtype_code(dtype))
    return out


def attn_fwd(q, k, v, scale: float, causal: bool, dtype):
    """Naive fp64 attention on BHSD inputs. Returns (O [B,H,S,D], LSE [B,H,S]) float64."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H, S, D = qb.shape
    o = np.empty((B, H, S, D), dtype=np.float64)
    lse = np.empty((B, H, S), dtype=np.float64)
    rc = lib.oracle_attn_fwd(_ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16),
                             _ptr(vb, ctypes.c_uint16), B, H, S, D, float(np.float32(scale)),
                             int(bool(causal)), _dtype_code(dtype),
                             _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd failed with {rc}")
    return o, lse


def attn_rows(q, k, v, scale: float, causal: bool, dtype, bh_idx, row_idx):
    """The definition for selected rows only. Returns (O [n,D], LSE [n]) float64."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H, S, D = qb.shape
    bh = np.ascontiguousarray(bh_idx, dtype=np.int64)
    ri = np.ascontiguousarray(row_idx, dtype=np.int64)
    n = bh.size
    o = np.empty((n, D), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    rc = lib.oracle_attn_rows(_ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16),
                              _ptr(vb, ctypes.c_uint16), B, H, S, D, float(np.float32(scale)),
                              int(bool(causal)), _dtype_code(dtype),
                              _ptr(bh, ctypes.c_int64), _ptr(ri, ctypes.c_int64), n,
                              _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_rows failed with {rc}")
    return o, lse


def attn_fwd_gen(q, k, v, scale: float, causal: bool, dtype):
    """Naive fp64 attention with Sq = q.shape[2] queries and Sk = k.shape[2] keys
    (contiguous BHSD); causal means query i sees keys j <= i + Sk - Sq."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H, Sq, D = qb.shape
    Sk = kb.shape[2]
    if kb.shape != (B, H, Sk, D) or vb.shape != kb.shape:
        raise ValueError("k and v must be [B, H, Sk, D] with q's B, H, D")
    o = np.empty((B, H, Sq, D), dtype=np.float64)
    lse = np.empty((B, H, Sq), dtype=np.float64)
    rc = lib.oracle_attn_fwd_gen(_ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16),
                                 _ptr(vb, ctypes.c_uint16), B, H, Sq, Sk, D, float(np.float32(scale)),
                                 int(bool(causal)), _dtype_code(dtype),
                                 _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_gen failed with {rc}")
    return o, lse


def attn_rows_gen(q, k, v, scale: float, causal: bool, dtype, bh_idx, row_idx):
    """attn_fwd_gen for selected (bh, query row) pairs. Returns (O [n,D], LSE [n])."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H, Sq, D = qb.shape
    Sk = kb.shape[2]
    bh = np.ascontiguousarray(bh_idx, dtype=np.int64)
    ri = np.ascontiguousarray(row_idx, dtype=np.int64)
    n = bh.size
    o = np.empty((n, D), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    rc = lib.oracle_attn_rows_gen(_ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16),
                                  _ptr(vb, ctypes.c_uint16), B, H, Sq, Sk, D, float(np.float32(scale)),
                                  int(bool(causal)), _dtype_code(dtype),
                                  _ptr(bh, ctypes.c_int64), _ptr(ri, ctypes.c_int64), n,
                                  _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_rows_gen failed with {rc}")
    return o, lse


def attn_fwd_masked(q, k, v, mask, scale: float, causal: bool, dtype):
    """attn_fwd_gen with an explicit boolean mask: ``mask`` broadcasts to
    [B, H, Sq, Sk] (a bool/uint8 tensor or array whose b and h dimensions may
    be 1); query i sees key j iff mask[..., i, j] (and the causal rule).  Rows
    that see no key give O = 0 and LSE = -inf."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H, Sq, D = qb.shape
    Sk = kb.shape[2]
    m = np.asarray(mask.cpu().numpy() if hasattr(mask, "cpu") else mask).astype(np.uint8)
    if m.ndim != 4 or m.shape[2:] != (Sq, Sk) or m.shape[0] not in (1, B) or m.shape[1] not in (1, H):
        raise ValueError("mask must be [B|1, H|1, Sq, Sk]")
    m = np.ascontiguousarray(m)
    sb = 0 if m.shape[0] == 1 else m.shape[1] * Sq * Sk
    sh = 0 if m.shape[1] == 1 else Sq * Sk
    o = np.empty((B, H, Sq, D))
    lse = np.empty((B, H, Sq))
    rc = lib.oracle_attn_fwd_masked(_ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
                                    B, H, Sq, Sk, D, float(np.float32(scale)), int(bool(causal)), _dtype_code(dtype),
                                    _ptr(m, ctypes.c_uint8), sb, sh, Sk, _ptr(o, ctypes.c_double),
                                    _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_masked failed with {rc}")
    return o, lse


def attn_bwd(q, k, v, dout, scale: float, causal: bool, dtype, magnitudes: bool = False):
    """fp64 gradients (dQ, dK, dV) of attention for the upstream gradient ``dout``
    (q, dout: [B,H,Sq,D]; k, v: [B,H,Sk,D]; bottom-right causal).  With
    ``magnitudes`` also returns the absolute-value sums (mag_dQ, mag_dK, mag_dV)
    that scale each element's 16-bit rounding error (see attn_oracle.c)."""
    lib = _load()
    qb, kb, vb, gb = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, H, Sq, D = qb.shape
    Sk = kb.shape[2]
    if gb.shape != qb.shape or kb.shape != (B, H, Sk, D) or vb.shape != kb.shape:
        raise ValueError("dout must be like q and k, v [B, H, Sk, D]")
    dq = np.empty((B, H, Sq, D))
    dk = np.empty((B, H, Sk, D))
    dv = np.empty((B, H, Sk, D))
    mags = tuple(np.empty(a.shape) for a in (dq, dk, dv)) if magnitudes else (None, None, None)
    fp = lambda a: _ptr(a, ctypes.c_double) if a is not None else None  # noqa: E731
    rc = lib.oracle_attn_bwd(_ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
                             _ptr(gb, ctypes.c_uint16), B, H, Sq, Sk, D, float(np.float32(scale)),
                             int(bool(causal)), _dtype_code(dtype), fp(dq), fp(dk), fp(dv),
                             fp(mags[0]), fp(mags[1]), fp(mags[2]))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_bwd failed with {rc}")
    return (dq, dk, dv) + (mags if magnitudes else ())


def attn_bwd_masked(q, k, v, dout, mask, scale: float, causal: bool, dtype, magnitudes: bool = False):
    """attn_bwd for the masked attention of attn_fwd_masked (mask [B|1, H|1, Sq, Sk])."""
    lib = _load()
    qb, kb, vb, gb = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, H, Sq, D = qb.shape
    Sk = kb.shape[2]
    m = np.asarray(mask.cpu().numpy() if hasattr(mask, "cpu") else mask).astype(np.uint8)
    if m.ndim != 4 or m.shape[2:] != (Sq, Sk) or m.shape[0] not in (1, B) or m.shape[1] not in (1, H):
        raise ValueError("mask must be [B|1, H|1, Sq, Sk]")
    m = np.ascontiguousarray(m)
    sb = 0 if m.shape[0] == 1 else m.shape[1] * Sq * Sk
    sh = 0 if m.shape[1] == 1 else Sq * Sk
    dq = np.empty((B, H, Sq, D))
    dk = np.empty((B, H, Sk, D))
    dv = np.empty((B, H, Sk, D))
    mags = tuple(np.empty(a.shape) for a in (dq, dk, dv)) if magnitudes else (None, None, None)
    fp = lambda a: _ptr(a, ctypes.c_double) if a is not None else None  # noqa: E731
    rc = lib.oracle_attn_bwd_masked(_ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
                                    _ptr(gb, ctypes.c_uint16), B, H, Sq, Sk, D, float(np.float32(scale)),
                                    int(bool(causal)), _dtype_code(dtype), _ptr(m, ctypes.c_uint8), sb, sh, Sk,
                                    fp(dq), fp(dk), fp(dv), fp(mags[0]), fp(mags[1]), fp(mags[2]))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_bwd_masked failed with {rc}")
    return (dq, dk, dv) + (mags if magnitudes else ())


def philox4x32_10(counter, key):
    """Philox4x32-10 of one 128-bit counter (4 words) under a 64-bit key (2 words)."""
    lib = _load()
    c = np.ascontiguousarray(counter, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    if c.shape != (4,) or k.shape != (2,):
        raise ValueError("counter: 4 words, key: 2 words")
    out = np.empty(4, dtype=np.uint32)
    lib.oracle_philox4x32_10(_ptr(c, ctypes.c_uint32), _ptr(k, ctypes.c_uint32), _ptr(out, ctypes.c_uint32))
    return out


def dropout_keep_mask(BH: int, Sq: int, Sk: int, p8: int, seed: int, offset: int) -> np.ndarray:
    """keep[bh, i, j] (1 = kept) of attention dropout with threshold p8 (1/256 units)."""
    lib = _load()
    keep = np.empty((BH, Sq, Sk), dtype=np.uint8)
    rc = lib.oracle_dropout_keep_mask(BH, Sq, Sk, int(p8), int(seed) & (2**64 - 1), int(offset) & 0xffffffff,
                                      _ptr(keep, ctypes.c_uint8))
    if rc != 0:
        raise RuntimeError(f"oracle_dropout_keep_mask failed with {rc}")
    return keep


def _mask_args(mask, B, H, Sq, Sk):
    """(array, strides over b, h, row) of a [B|1, H|1, Sq, Sk] mask, or (None, 0, 0, 0)."""
    if mask is None:
        return None, 0, 0, 0
    m = np.asarray(mask.cpu().numpy() if hasattr(mask, "cpu") else mask).astype(np.uint8)
    if m.ndim != 4 or m.shape[2:] != (Sq, Sk) or m.shape[0] not in (1, B) or m.shape[1] not in (1, H):
        raise ValueError("mask must be [B|1, H|1, Sq, Sk]")
    m = np.ascontiguousarray(m)
    return m, (0 if m.shape[0] == 1 else m.shape[1] * Sq * Sk), (0 if m.shape[1] == 1 else Sq * Sk), Sk


def attn_fwd_dropout(q, k, v, scale: float, causal: bool, dtype, p8: int, seed: int, offset: int, mask=None):
    """attn_fwd_gen with dropout after the softmax: weights kept by the Philox rule
    of attn_oracle.c (threshold p8 in 1/256 units), kept weights scaled by
    256 / (256 - p8); LSE of the undropped softmax.  ``mask`` (optional, as
    attn_fwd_masked's) restricts the keys each row sees."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H, Sq, D = qb.shape
    Sk = kb.shape[2]
    o = np.empty((B, H, Sq, D))
    lse = np.empty((B, H, Sq))
    m, sb, sh, si = _mask_args(mask, B, H, Sq, Sk)
    rc = lib.oracle_attn_fwd_dropout_masked(_ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16),
                                            _ptr(vb, ctypes.c_uint16), B, H, Sq, Sk, D, float(np.float32(scale)),
                                            int(bool(causal)), _dtype_code(dtype), int(p8), int(seed) & (2**64 - 1),
                                            int(offset) & 0xffffffff,
                                            _ptr(m, ctypes.c_uint8) if m is not None else None, sb, sh, si,
                                            _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_dropout failed with {rc}")
    return o, lse


def attn_rows_dropout(q, k, v, scale: float, causal: bool, dtype, p8: int, seed: int, offset: int, bh_idx, row_idx):
    """attn_fwd_dropout for selected (bh, query row) pairs. Returns (O [n,D], LSE [n])."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H, Sq, D = qb.shape
    Sk = kb.shape[2]
    bh = np.ascontiguousarray(bh_idx, dtype=np.int64)
    ri = np.ascontiguousarray(row_idx, dtype=np.int64)
    n = bh.size
    o = np.empty((n, D))
    lse = np.empty((n,))
    rc = lib.oracle_attn_rows_dropout(_ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
                                      B, H, Sq, Sk, D, float(np.float32(scale)), int(bool(causal)),
                                      _dtype_code(dtype), int(p8), int(seed) & (2**64 - 1), int(offset) & 0xffffffff,
                                      _ptr(bh, ctypes.c_int64), _ptr(ri, ctypes.c_int64), n,
                                      _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_rows_dropout failed with {rc}")
    return o, lse


def attn_bwd_dropout(q, k, v, dout, scale: float, causal: bool, dtype, p8: int, seed: int, offset: int,
                     magnitudes: bool = False, mask=None):
    """attn_bwd for the attention with dropout (and optional mask) of attn_fwd_dropout."""
    lib = _load()
    qb, kb, vb, gb = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, H, Sq, D = qb.shape
    Sk = kb.shape[2]
    dq = np.empty((B, H, Sq, D))
    dk = np.empty((B, H, Sk, D))
    dv = np.empty((B, H, Sk, D))
    mags = tuple(np.empty(a.shape) for a in (dq, dk, dv)) if magnitudes else (None, None, None)
    fp = lambda a: _ptr(a, ctypes.c_double) if a is not None else None  # noqa: E731
    m, sb, sh, si = _mask_args(mask, B, H, Sq, Sk)
    rc = lib.oracle_attn_bwd_dropout_masked(_ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16),
                                            _ptr(vb, ctypes.c_uint16), _ptr(gb, ctypes.c_uint16), B, H, Sq, Sk, D,
                                            float(np.float32(scale)), int(bool(causal)), _dtype_code(dtype), int(p8),
                                            int(seed) & (2**64 - 1), int(offset) & 0xffffffff,
                                            _ptr(m, ctypes.c_uint8) if m is not None else None, sb, sh, si,
                                            fp(dq), fp(dk), fp(dv), fp(mags[0]), fp(mags[1]), fp(mags[2]))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_bwd_dropout failed with {rc}")
    return (dq, dk, dv) + (mags if magnitudes else ())


def attn_tiled(q, k, v, scale: float, causal: bool, dtype, Br: int, Bc: int, form: int = 0):
    """Tiled online-softmax reference (form 0 deferred /l, form 1 per-step normalised)."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H, S, D = qb.shape
    o = np.empty((B, H, S, D), dtype=np.float64)
    lse = np.empty((B, H, S), dtype=np.float64)
    rc = lib.oracle_attn_tiled(_ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16),
                               _ptr(vb, ctypes.c_uint16), B, H, S, D, float(np.float32(scale)),
                               int(bool(causal)), _dtype_code(dtype), int(Br), int(Bc), int(form),
                               _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_tiled failed with {rc}")
    return o, lse


def attn_probs(q, k, scale: float, causal: bool, dtype, bh: int = 0) -> np.ndarray:
    """Softmax matrix P [S,S] of head ``bh`` (flattened b*H+h)."""
    lib = _load()
    qb, kb = _bits(q), _bits(k)
    B, H, S, D = qb.shape
    p = np.empty((S, S), dtype=np.float64)
    rc = lib.oracle_attn_probs(_ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16), B, H, S, D,
                               float(np.float32(scale)), int(bool(causal)), _dtype_code(dtype),
                               int(bh), _ptr(p, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_probs failed with {rc}")
    return p


def causal_tile_count(S: int, BM: int, BN: int):
    """(total, computed, skipped) tile pairs of a causal S x S problem, by enumeration."""
    lib = _load()
    t, c, s = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    lib.oracle_causal_tile_count(int(S), int(BM), int(BN), ctypes.byref(t), ctypes.byref(c),
                                 ctypes.byref(s))
    return t.value, c.value, s.value


def num_threads() -> int:
    return int(_load().oracle_num_threads())

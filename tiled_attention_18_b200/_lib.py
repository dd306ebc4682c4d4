"""ctypes binding of libfa.so (include/fa.h): argument marshalling only.

Every step of the attention computation runs in the CUDA kernels of
libfa.so.  If the library is missing or cannot be loaded, every call raises:
there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa.so")

FA_FP16 = 0
FA_BF16 = 1

FA_OK = 0
FA_ERR_NULL = -1
FA_ERR_SHAPE = -2
FA_ERR_HEADDIM = -3
FA_ERR_DTYPE = -4
FA_ERR_ALIGN = -5
FA_ERR_ARCH = -6
FA_ERR_LAUNCH = -7
FA_ERR_TIMEOUT = -8
FA_ERR_SCALE = -9
FA_ERR_ARG = -10
FA_ERR_PTR = -11
FA_ERR_STRIDE = -12
FA_ERR_WORKSPACE = -13
FA_ERR_LIMIT = -14

_LL3 = ctypes.POINTER(ctypes.c_longlong)

# (name, restype, argtypes) of every symbol include/fa.h declares
SIGNATURES = [
    ("fa_fwd", ctypes.c_int,
     [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
      ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
      ctypes.c_int, ctypes.c_void_p]),
    ("fa_fwd_noalloc", ctypes.c_int,
     [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
      ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
      ctypes.c_int, ctypes.c_void_p]),
    ("fa_fwd_ex", ctypes.c_int,
     [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
      ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
      _LL3, _LL3, _LL3, _LL3, ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    ("fa_fwd_mask", ctypes.c_int,
     [ctypes.c_void_p] * 5 + [ctypes.c_int] * 5 + [ctypes.c_void_p, _LL3, ctypes.c_float, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_void_p]),
    ("fa_bwd_workspace_size", ctypes.c_longlong, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    ("fa_bwd", ctypes.c_int,
     [ctypes.c_void_p] * 10 + [ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                               ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                               ctypes.c_void_p]),
    ("fa_bwd_ex", ctypes.c_int,
     [ctypes.c_void_p] * 10 + [ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                               ctypes.c_int] + [_LL3] * 8 + [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                           ctypes.c_void_p]),
    ("fa_bwd_mask", ctypes.c_int,
     [ctypes.c_void_p] * 10 + [ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                               ctypes.c_int, ctypes.c_void_p, _LL3, ctypes.c_float, ctypes.c_int, ctypes.c_int,
                               ctypes.c_int, ctypes.c_void_p]),
    ("fa_fwd_dropout", ctypes.c_int,
     [ctypes.c_void_p] * 5 + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_int, ctypes.c_float, ctypes.c_ulonglong,
                                                ctypes.c_uint, ctypes.c_int, ctypes.c_void_p]),
    ("fa_bwd_dropout", ctypes.c_int,
     [ctypes.c_void_p] * 10 + [ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                               ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_float, ctypes.c_ulonglong,
                               ctypes.c_uint, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    ("fa_forward", ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    ("fa_backward", ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    ("fa_accumulate", ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int, ctypes.c_void_p]),
    ("fa_merge_partial", ctypes.c_int,
     [ctypes.c_void_p] * 4 + [ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    ("fa_merge_finalize", ctypes.c_int,
     [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int, ctypes.c_void_p]),
    ("fa_check_status", ctypes.c_int, [ctypes.c_void_p]),
    ("fa_last_timeout_site", ctypes.c_int, []),
    ("fa_last_cuda_error", ctypes.c_int, [ctypes.POINTER(ctypes.c_char_p)]),
    ("fa_selftest_timeout", ctypes.c_int, [ctypes.c_void_p]),
    ("fa_status_string", ctypes.c_char_p, [ctypes.c_int]),
    ("fa_version", ctypes.c_int, []),
    ("fa_num_units", ctypes.c_longlong, [ctypes.c_int, ctypes.c_int, ctypes.c_int]),
]

_lock = threading.Lock()
_lib = None


class FaError(RuntimeError):
    def __init__(self, status: int, what: str = "fa_fwd"):
        self.status = status
        msg = f"{what} failed: {status} ({status_string(status)})"
        if status == FA_ERR_LAUNCH:
            # the failing CUDA call of this thread, as the library recorded it
            try:
                code, site = fa_last_cuda_error()
                msg += f"; CUDA error {code} in {site}"
            except OSError:
                pass
        super().__init__(msg)


def load() -> ctypes.CDLL:
    """Load libfa.so (raises OSError if it is missing: build it with
    ``python -m tiled_attention_18_b200.build``)."""
    global _lib
    lib = _lib
    if lib is not None:  # loaded: no lock on the per-call path
        return lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise OSError(f"{LIB_PATH} not found; build it with `python -m tiled_attention_18_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def fa_fwd(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int, H: int, S: int, D: int,
           scale: float, causal: int, dtype: int, stream: int) -> int:
    """Raw C call: device pointers as integers, returns the fa_status code."""
    return int(load().fa_fwd(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, S, D, float(scale), int(causal),
                             int(dtype), stream))


def fa_fwd_noalloc(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int, H: int, S: int,
                   D: int, scale: float, causal: int, dtype: int, stream: int) -> int:
    """Raw C call of the variant that allocates no device memory (see include/fa.h)."""
    return int(load().fa_fwd_noalloc(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, S, D, float(scale),
                                     int(causal), int(dtype), stream))


_LL3_CACHE = {}


def _strides(st):
    """A (b, h, s) stride triple as a C array (arrays are read-only to the library,
    so one array per distinct triple is kept and reused)."""
    if st is None:
        return None
    key = tuple(st)
    arr = _LL3_CACHE.get(key)
    if arr is None:
        vals = [int(x) for x in key]
        if len(vals) != 3:
            raise ValueError("a stride triple (b, h, s) is expected")
        arr = (ctypes.c_longlong * 3)(*vals)
        if len(_LL3_CACHE) < 4096:
            _LL3_CACHE[key] = arr
    return arr


def fa_fwd_ex(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int, H: int, Sq: int, Sk: int,
              D: int, q_stride, k_stride, v_stride, o_stride, scale: float, causal: int, dtype: int,
              stream: int) -> int:
    """Raw C call of the general-shape entry: each *_stride is a (b, h, s) element-stride
    triple or None for contiguous BHSD."""
    return int(load().fa_fwd_ex(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, Sq, Sk, D, _strides(q_stride),
                                _strides(k_stride), _strides(v_stride), _strides(o_stride), float(scale),
                                int(causal), int(dtype), stream))


def fa_fwd_mask(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int, H: int, Sq: int, Sk: int,
                D: int, mask_ptr: int, mask_stride, scale: float, causal: int, dtype: int, stream: int) -> int:
    """Raw C call of the explicit-mask forward: mask_stride is a (b, h, row) element-stride triple."""
    return int(load().fa_fwd_mask(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, Sq, Sk, D, mask_ptr,
                                  _strides(mask_stride), float(scale), int(causal), int(dtype), stream))


def fa_bwd_workspace_size(B: int, H: int, Sq: int, D: int) -> int:
    return int(load().fa_bwd_workspace_size(B, H, Sq, D))


def fa_bwd(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, do_ptr: int, lse_ptr: int, dq_ptr: int, dk_ptr: int,
           dv_ptr: int, ws_ptr: int, ws_bytes: int, B: int, H: int, Sq: int, Sk: int, D: int, scale: float,
           causal: int, deterministic: int, dtype: int, stream: int) -> int:
    """Raw C call of the backward pass (see include/fa.h)."""
    return int(load().fa_bwd(q_ptr, k_ptr, v_ptr, o_ptr, do_ptr, lse_ptr, dq_ptr, dk_ptr, dv_ptr, ws_ptr,
                             int(ws_bytes), B, H, Sq, Sk, D, float(scale), int(causal), int(deterministic),
                             int(dtype), stream))


def fa_bwd_ex(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, do_ptr: int, lse_ptr: int, dq_ptr: int, dk_ptr: int,
              dv_ptr: int, ws_ptr: int, ws_bytes: int, B: int, H: int, Sq: int, Sk: int, D: int, q_stride, k_stride,
              v_stride, o_stride, do_stride, dq_stride, dk_stride, dv_stride, scale: float, causal: int,
              deterministic: int, dtype: int, stream: int) -> int:
    """Raw C call of the strided backward pass: each stride argument is a (b, h, s)
    element-stride triple or None (contiguous)."""
    return int(load().fa_bwd_ex(q_ptr, k_ptr, v_ptr, o_ptr, do_ptr, lse_ptr, dq_ptr, dk_ptr, dv_ptr, ws_ptr,
                                int(ws_bytes), B, H, Sq, Sk, D, _strides(q_stride), _strides(k_stride),
                                _strides(v_stride), _strides(o_stride), _strides(do_stride), _strides(dq_stride),
                                _strides(dk_stride), _strides(dv_stride), float(scale), int(causal),
                                int(deterministic), int(dtype), stream))


def fa_bwd_mask(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, do_ptr: int, lse_ptr: int, dq_ptr: int,
                dk_ptr: int, dv_ptr: int, ws_ptr: int, ws_bytes: int, B: int, H: int, Sq: int, Sk: int, D: int,
                mask_ptr: int, mask_stride, scale: float, causal: int, deterministic: int, dtype: int,
                stream: int) -> int:
    """Raw C call of the masked backward pass (see include/fa.h)."""
    return int(load().fa_bwd_mask(q_ptr, k_ptr, v_ptr, o_ptr, do_ptr, lse_ptr, dq_ptr, dk_ptr, dv_ptr, ws_ptr,
                                  int(ws_bytes), B, H, Sq, Sk, D, mask_ptr, _strides(mask_stride), float(scale),
                                  int(causal), int(deterministic), int(dtype), stream))


def fa_fwd_dropout(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int, H: int, Sq: int, Sk: int,
                   D: int, scale: float, causal: int, dropout_p: float, seed: int, offset: int, dtype: int,
                   stream: int) -> int:
    """Raw C call of the forward pass with dropout (see include/fa.h)."""
    return int(load().fa_fwd_dropout(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, Sq, Sk, D, float(scale), int(causal),
                                     float(dropout_p), int(seed) & (2**64 - 1), int(offset) & 0xffffffff, int(dtype),
                                     stream))


def fa_bwd_dropout(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, do_ptr: int, lse_ptr: int, dq_ptr: int,
                   dk_ptr: int, dv_ptr: int, ws_ptr: int, ws_bytes: int, B: int, H: int, Sq: int, Sk: int, D: int,
                   scale: float, causal: int, dropout_p: float, seed: int, offset: int, deterministic: int,
                   dtype: int, stream: int) -> int:
    """Raw C call of the backward pass with dropout (see include/fa.h)."""
    return int(load().fa_bwd_dropout(q_ptr, k_ptr, v_ptr, o_ptr, do_ptr, lse_ptr, dq_ptr, dk_ptr, dv_ptr, ws_ptr,
                                     int(ws_bytes), B, H, Sq, Sk, D, float(scale), int(causal), float(dropout_p),
                                     int(seed) & (2**64 - 1), int(offset) & 0xffffffff, int(deterministic),
                                     int(dtype), stream))


_LLP = ctypes.POINTER(ctypes.c_longlong)


class FwdParams(ctypes.Structure):
    """fa_fwd_params of include/fa.h (same field order and C types)."""
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("o", ctypes.c_void_p),
                ("lse", ctypes.c_void_p), ("B", ctypes.c_int), ("H", ctypes.c_int), ("Sq", ctypes.c_int),
                ("Sk", ctypes.c_int), ("D", ctypes.c_int), ("q_stride", _LLP), ("k_stride", _LLP),
                ("v_stride", _LLP), ("o_stride", _LLP), ("mask", ctypes.c_void_p), ("mask_stride", _LLP),
                ("dropout_p", ctypes.c_float), ("seed", ctypes.c_ulonglong), ("offset", ctypes.c_uint),
                ("scale", ctypes.c_float), ("causal", ctypes.c_int), ("dtype", ctypes.c_int),
                ("block_n", ctypes.c_int), ("q_tiles", ctypes.c_int)]


class BwdParams(ctypes.Structure):
    """fa_bwd_params of include/fa.h (same field order and C types)."""
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("o", ctypes.c_void_p),
                ("dout", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("dq", ctypes.c_void_p),
                ("dk", ctypes.c_void_p), ("dv", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_longlong), ("B", ctypes.c_int), ("H", ctypes.c_int),
                ("Sq", ctypes.c_int), ("Sk", ctypes.c_int), ("D", ctypes.c_int), ("q_stride", _LLP),
                ("k_stride", _LLP), ("v_stride", _LLP), ("o_stride", _LLP), ("do_stride", _LLP),
                ("dq_stride", _LLP), ("dk_stride", _LLP), ("dv_stride", _LLP), ("mask", ctypes.c_void_p),
                ("mask_stride", _LLP), ("dropout_p", ctypes.c_float), ("seed", ctypes.c_ulonglong),
                ("offset", ctypes.c_uint), ("scale", ctypes.c_float), ("causal", ctypes.c_int),
                ("deterministic", ctypes.c_int), ("dtype", ctypes.c_int)]


def _params(cls, keep: list, **kw):
    """A params struct; stride triples become C arrays kept alive in ``keep``."""
    p = cls()
    for name, val in kw.items():
        if name.endswith("stride"):
            if val is not None:
                arr = (ctypes.c_longlong * 3)(*[int(x) for x in val])
                keep.append(arr)
                setattr(p, name, ctypes.cast(arr, _LLP))
        elif name == "seed":
            p.seed = int(val) & (2**64 - 1)
        elif name == "offset":
            p.offset = int(val) & 0xffffffff
        else:
            setattr(p, name, val)
    return p


def fa_forward(stream: int, **kw) -> int:
    """fa_forward with the fields of fa_fwd_params as keyword arguments (pointers
    as ints, strides as triples or None)."""
    keep: list = []
    p = _params(FwdParams, keep, **kw)
    return int(load().fa_forward(ctypes.byref(p), stream))


def fa_backward(stream: int, **kw) -> int:
    """fa_backward with the fields of fa_bwd_params as keyword arguments."""
    keep: list = []
    p = _params(BwdParams, keep, **kw)
    return int(load().fa_backward(ctypes.byref(p), stream))


def fa_accumulate(acc_ptr: int, x_ptr: int, n: int, dtype: int, stream: int) -> int:
    """Raw C call: acc (fp32) += x (16-bit) over n values."""
    return int(load().fa_accumulate(acc_ptr, x_ptr, int(n), int(dtype), stream))


def fa_merge_partial(o_acc_ptr: int, lse_acc_ptr: int, o_part_ptr: int, lse_part_ptr: int, rows: int, D: int,
                     dtype: int, stream: int) -> int:
    return int(load().fa_merge_partial(o_acc_ptr, lse_acc_ptr, o_part_ptr, lse_part_ptr, int(rows), D, int(dtype),
                                       stream))


def fa_merge_finalize(o_acc_ptr: int, o_ptr: int, n: int, dtype: int, stream: int) -> int:
    return int(load().fa_merge_finalize(o_acc_ptr, o_ptr, int(n), int(dtype), stream))


def fa_check_status(stream: int = 0) -> int:
    return int(load().fa_check_status(stream))


def fa_last_timeout_site() -> int:
    return int(load().fa_last_timeout_site())


def fa_last_cuda_error():
    """(code, call name) of the CUDA failure behind this thread's latest FA_ERR_LAUNCH; (0, "") if none."""
    site = ctypes.c_char_p()
    code = int(load().fa_last_cuda_error(ctypes.byref(site)))
    return code, (site.value or b"").decode()


def fa_selftest_timeout(stream: int = 0) -> int:
    return int(load().fa_selftest_timeout(stream))


def fa_status_string(status: int) -> str:
    return load().fa_status_string(int(status)).decode()


def status_string(status: int) -> str:
    try:
        return fa_status_string(status)
    except OSError:
        return "libfa.so not loaded"


def fa_version() -> int:
    return int(load().fa_version())


def fa_num_units(B: int, H: int, S: int) -> int:
    return int(load().fa_num_units(B, H, S))

"""C-ABI checks that need no GPU: the library loads, exports every symbol
include/fa.h declares, and rejects invalid arguments before any CUDA call."""
import ctypes
import math
import os
import re

import pytest

import tiled_attention_18_b200 as fa
from tiled_attention_18_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "fa.h")) as f:
        text = f.read()
    return re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    from tiled_attention_18_b200 import build
    build.build()
    return fa.load()


def test_header_declares_the_entry_points():
    syms = _declared_symbols()
    assert set(syms) == {name for name, _, _ in _lib.SIGNATURES}


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_symbols():
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr), name


def test_status_enum_matches_header(lib):
    with open(os.path.join(ROOT, "include", "fa.h")) as f:
        text = f.read()
    codes = dict((k, int(v)) for k, v in re.findall(r"(FA_(?:OK|ERR_\w+))\s*=\s*(-?\d+)", text))
    for name, value in codes.items():
        assert getattr(_lib, name) == value, name
        assert fa.fa_status_string(value) not in ("", "unknown status")
    assert fa.fa_status_string(12345) == "unknown status"


def test_version_and_units(lib):
    assert fa.fa_version() == 100
    assert fa.fa_num_units(1, 32, 16384) == 32 * 64
    assert fa.fa_num_units(2, 12, 2048) == 24 * 8
    assert fa.fa_num_units(1, 1, 257) == 2
    assert fa.fa_num_units(1, 1, 256) == 1
    assert fa.fa_num_units(0, 4, 100) == 0
    assert fa.fa_num_units(1, 1, -1) == _lib.FA_ERR_SHAPE


A = 0x10000  # an aligned, non-null address (never dereferenced: checks fail first)


@pytest.mark.parametrize("args,code", [
    (dict(B=-1), _lib.FA_ERR_SHAPE),
    (dict(S=-5), _lib.FA_ERR_SHAPE),
    (dict(D=96), _lib.FA_ERR_HEADDIM),
    (dict(D=512), _lib.FA_ERR_HEADDIM),
    (dict(dtype=2), _lib.FA_ERR_DTYPE),
    (dict(scale=0.0), _lib.FA_ERR_SCALE),
    (dict(scale=-1.0), _lib.FA_ERR_SCALE),
    (dict(scale=math.nan), _lib.FA_ERR_SCALE),
    (dict(scale=math.inf), _lib.FA_ERR_SCALE),
    (dict(causal=2), _lib.FA_ERR_ARG),
    (dict(q=0), _lib.FA_ERR_NULL),
    (dict(lse=0), _lib.FA_ERR_NULL),
    (dict(o=A + 8), _lib.FA_ERR_ALIGN),
    (dict(lse=A + 2), _lib.FA_ERR_ALIGN),
    (dict(B=1 << 16, H=1 << 16), _lib.FA_ERR_SHAPE),
])
def test_invalid_arguments_rejected_before_launch(lib, args, code):
    a = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=2, S=128, D=64, scale=0.125, causal=0, dtype=0, stream=0)
    a.update(args)
    st = fa.fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["S"], a["D"], a["scale"],
                   a["causal"], a["dtype"], a["stream"])
    assert st == code


def test_empty_problem_is_a_noop(lib):
    for B, H, S in ((0, 2, 128), (1, 0, 128), (1, 2, 0)):
        assert fa.fa_fwd(0, 0, 0, 0, 0, B, H, S, 64, 0.125, 0, 0, 0) == _lib.FA_OK


def test_no_device_is_reported_not_faulted(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    st = fa.fa_fwd(A, A, A, A, A, 1, 2, 128, 64, 0.125, 0, 0, 0)
    assert st == _lib.FA_ERR_LAUNCH


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(OSError):
        _lib.load()


@pytest.mark.parametrize("args,code", [
    (dict(Sq=-1), _lib.FA_ERR_SHAPE),
    (dict(Sk=-1), _lib.FA_ERR_SHAPE),
    (dict(Sk=0), _lib.FA_ERR_SHAPE),                      # a query would see no key
    (dict(Sq=200, Sk=100, causal=1), _lib.FA_ERR_SHAPE),  # bottom-right mask: first rows see nothing
    (dict(Sk=(1 << 31) - 100), _lib.FA_ERR_SHAPE),
    (dict(D=32), _lib.FA_ERR_HEADDIM),
    (dict(dtype=-1), _lib.FA_ERR_DTYPE),
    (dict(scale=0.0), _lib.FA_ERR_SCALE),
    (dict(causal=-1), _lib.FA_ERR_ARG),
    (dict(v=0), _lib.FA_ERR_NULL),
    (dict(qs=(128 * 64 * 2, 64, 2 * 64 + 4)), _lib.FA_ERR_STRIDE),   # s stride not 16 bytes
    (dict(ks=(0, 64, 128)), _lib.FA_ERR_STRIDE),                     # zero over B = 2
    (dict(vs=(-8, 64, 128)), _lib.FA_ERR_STRIDE),
    (dict(os=(1 << 36, 64, 128)), _lib.FA_ERR_STRIDE),
    (dict(k=A + 2), _lib.FA_ERR_ALIGN),
])
def test_fa_fwd_ex_invalid_arguments(lib, args, code):
    a = dict(q=A, k=A, v=A, o=A, lse=A, B=2, H=3, Sq=100, Sk=300, D=64, qs=None, ks=None, vs=None, os=None,
             scale=0.125, causal=0, dtype=1)
    a.update(args)
    st = fa.fa_fwd_ex(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Sq"], a["Sk"], a["D"],
                      a["qs"], a["ks"], a["vs"], a["os"], a["scale"], a["causal"], a["dtype"], 0)
    assert st == code


def test_fa_fwd_ex_stride_over_unit_extent_is_ignored(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    # B = 1 and H = 1: the (invalid) b and h strides are never used; the call
    # gets past every argument check and stops at the missing device
    st = fa.fa_fwd_ex(A, A, A, A, A, 1, 1, 64, 64, 64, (3, -5, 64), (0, 0, 64), None, None, 0.125, 1, 0, 0)
    assert st == _lib.FA_ERR_LAUNCH


def test_fa_fwd_ex_empty_problems(lib):
    for B, H, Sq, Sk in ((0, 2, 10, 10), (1, 0, 10, 10), (1, 2, 0, 10), (1, 2, 0, 0)):
        assert fa.fa_fwd_ex(0, 0, 0, 0, 0, B, H, Sq, Sk, 64, None, None, None, None, 0.1, 1, 0, 0) == _lib.FA_OK


def test_bwd_workspace_size(lib):
    assert fa.fa_bwd_workspace_size(0, 4, 100, 64) == 0
    assert fa.fa_bwd_workspace_size(1, 1, -1, 64) == _lib.FA_ERR_SHAPE
    assert fa.fa_bwd_workspace_size(1, 1, 10, 96) == _lib.FA_ERR_HEADDIM
    # dQ accumulator (fp32) + two padded fp32 row arrays + turn counters + 256-byte
    # scheduler counter + dK/dV partial sums, 256-aligned parts
    B, H, S, D = 2, 3, 300, 128
    up = lambda x: -(-x // 256) * 256  # noqa: E731
    acc = up(B * H * S * D * 4)
    rows = up(B * H * 384 * 4)
    flags = up(B * H * 5 * 4 * 4)
    kv = up(2 * B * H * 128 * D * 4)  # fp32 dK/dV partial sums of a split query range (<= 128 keys)
    assert fa.fa_bwd_workspace_size(B, H, S, D) == acc + 2 * rows + flags + 256 + kv
    # D = 256: twice the dQ accumulator and a turn counter per half of the head dimension
    acc = up(B * H * S * 256 * 4)
    flags = up(B * H * 5 * 2 * 4 * 4)
    kv = up(2 * B * H * 128 * 256 * 4)
    assert fa.fa_bwd_workspace_size(B, H, S, 256) == acc + 2 * rows + flags + 256 + kv


@pytest.mark.parametrize("args,code", [
    (dict(Sq=-1), _lib.FA_ERR_SHAPE),
    (dict(Sk=0), _lib.FA_ERR_SHAPE),
    (dict(Sq=300, Sk=200, causal=1), _lib.FA_ERR_SHAPE),
    (dict(D=512), _lib.FA_ERR_HEADDIM),
    (dict(dtype=3), _lib.FA_ERR_DTYPE),
    (dict(scale=math.nan), _lib.FA_ERR_SCALE),
    (dict(causal=5), _lib.FA_ERR_ARG),
    (dict(det=2), _lib.FA_ERR_ARG),
    (dict(dout=0), _lib.FA_ERR_NULL),
    (dict(dq=0), _lib.FA_ERR_NULL),
    (dict(ws=0), _lib.FA_ERR_WORKSPACE),
    (dict(ws=A + 128), _lib.FA_ERR_WORKSPACE),
    (dict(ws_bytes=100), _lib.FA_ERR_WORKSPACE),
    (dict(dk=A + 8), _lib.FA_ERR_ALIGN),
    (dict(lse=A + 1), _lib.FA_ERR_ALIGN),
])
def test_fa_bwd_invalid_arguments(lib, args, code):
    a = dict(q=A, k=A, v=A, o=A, dout=A, lse=A, dq=A, dk=A, dv=A, ws=A, ws_bytes=1 << 30, B=1, H=2, Sq=100, Sk=300,
             D=64, scale=0.125, causal=0, det=0, dtype=0)
    a.update(args)
    st = fa.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["dout"], a["lse"], a["dq"], a["dk"], a["dv"], a["ws"],
                   a["ws_bytes"], a["B"], a["H"], a["Sq"], a["Sk"], a["D"], a["scale"], a["causal"], a["det"],
                   a["dtype"], 0)
    assert st == code


def test_fa_bwd_empty_problems(lib):
    for B, H, Sq, Sk in ((0, 2, 10, 10), (1, 0, 10, 10), (1, 2, 0, 0)):
        assert fa.fa_bwd(0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, B, H, Sq, Sk, 64, 0.1, 0, 0, 0, 0) == _lib.FA_OK


@pytest.mark.parametrize("args,code", [
    (dict(mask=0), _lib.FA_ERR_NULL),
    (dict(ms=None), _lib.FA_ERR_NULL),
    (dict(ms=(0, 0, 100)), _lib.FA_ERR_STRIDE),         # row stride below Sk
    (dict(ms=(0, 0, 328)), _lib.FA_ERR_STRIDE),         # row stride not a multiple of 16
    (dict(ms=(-16, 0, 336)), _lib.FA_ERR_STRIDE),
    (dict(ms=(8, 0, 336)), _lib.FA_ERR_STRIDE),
    (dict(mask=A + 4), _lib.FA_ERR_ALIGN),
    (dict(D=80), _lib.FA_ERR_HEADDIM),
    (dict(D=512), _lib.FA_ERR_HEADDIM),               # the mask is fused into the D = 64/128/256 kernels
    (dict(Sq=400, Sk=300, causal=1), _lib.FA_ERR_SHAPE),
])
def test_fa_fwd_mask_invalid_arguments(lib, args, code):
    a = dict(q=A, k=A, v=A, o=A, lse=A, B=2, H=3, Sq=100, Sk=330, D=64, mask=A, ms=(0, 0, 336), scale=0.125,
             causal=0, dtype=1)
    a.update(args)
    st = fa.fa_fwd_mask(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Sq"], a["Sk"], a["D"], a["mask"],
                        a["ms"], a["scale"], a["causal"], a["dtype"], 0)
    assert st == code


def test_merge_entries_reject_bad_arguments(lib):
    assert fa.fa_merge_partial(A, A, A, A, -1, 64, 1, 0) == _lib.FA_ERR_SHAPE
    assert fa.fa_merge_partial(A, A, A, A, 10, 0, 1, 0) == _lib.FA_ERR_HEADDIM
    assert fa.fa_merge_partial(A, A, A, A, 10, 64, 5, 0) == _lib.FA_ERR_DTYPE
    assert fa.fa_merge_partial(0, A, A, A, 10, 64, 1, 0) == _lib.FA_ERR_NULL
    assert fa.fa_merge_partial(A + 2, A, A, A, 10, 64, 1, 0) == _lib.FA_ERR_ALIGN
    assert fa.fa_merge_partial(0, 0, 0, 0, 0, 64, 1, 0) == _lib.FA_OK
    assert fa.fa_merge_finalize(A, A, -1, 1, 0) == _lib.FA_ERR_SHAPE
    assert fa.fa_merge_finalize(A, A + 1, 10, 1, 0) == _lib.FA_ERR_ALIGN
    assert fa.fa_merge_finalize(0, 0, 0, 1, 0) == _lib.FA_OK


def test_dropout_entries_reject_bad_arguments(lib):
    ok = dict(B=1, H=1, Sq=128, Sk=128, D=128)
    args = lambda p, D=128, B=1: (A, A, A, A, A, B, 1, 128, 128, D, 0.1, 0, p, 1, 0, 1, 0)  # noqa: E731
    for p in (-0.1, float("nan"), float("inf"), 1.0, 255.5 / 256):
        assert fa.fa_fwd_dropout(*args(p)) == _lib.FA_ERR_ARG, p
    assert fa.fa_fwd_dropout(*args(0.2, D=512)) == _lib.FA_ERR_HEADDIM
    assert fa.fa_fwd_dropout(*args(0.2, B=0)) == _lib.FA_OK  # empty problem, nothing launched
    assert fa.fa_fwd_dropout(*args(0.2, B=-1)) == _lib.FA_ERR_SHAPE
    bargs = lambda p, D=128: (A,) * 10 + (1 << 20, 1, 1, 128, 128, D, 0.1, 0, p, 1, 0, 0, 1, 0)  # noqa: E731
    for p in (-0.5, float("nan"), 1.0):
        assert fa.fa_bwd_dropout(*bargs(p)) == _lib.FA_ERR_ARG, p
    assert fa.fa_bwd_dropout(*bargs(0.1, D=512)) == _lib.FA_ERR_HEADDIM
    assert ok  # the shapes above are otherwise valid


def test_bwd_ex_rejects_bad_strides(lib):
    def call(B=1, H=2, Sq=128, Sk=128, strides=(None,) * 8):
        return fa.fa_bwd_ex(A, A, A, A, A, A, A, A, A, A, 1 << 30, B, H, Sq, Sk, 64, *strides, 0.1, 0, 0, 1, 0)
    for bad in ((7, 64, 64), (0, 64, 64), (-8, 64, 64), (1 << 36, 64, 64)):
        for t in range(8):
            st = [None] * 8
            st[t] = bad
            assert call(B=2, strides=st) == _lib.FA_ERR_STRIDE, (t, bad)
    # a stride over an extent of 1 is ignored (B = 1: the batch stride)
    st = [None] * 8
    st[0] = (3, 2 * 128 * 64, 64)
    assert call(Sq=0, Sk=0, strides=st) == _lib.FA_OK
    # no query: dK/dV are zeroed as contiguous blocks, so their strides must be NULL
    st = [None] * 8
    st[6] = (2 * 128 * 64, 128 * 64, 64)
    assert call(Sq=0, strides=st) == _lib.FA_ERR_STRIDE


def test_accumulate_rejects_bad_arguments(lib):
    assert fa.fa_accumulate(A, A, -1, 1, 0) == _lib.FA_ERR_SHAPE
    assert fa.fa_accumulate(A, A, 10, 7, 0) == _lib.FA_ERR_DTYPE
    assert fa.fa_accumulate(0, A, 10, 1, 0) == _lib.FA_ERR_NULL
    assert fa.fa_accumulate(A + 2, A, 10, 1, 0) == _lib.FA_ERR_ALIGN
    assert fa.fa_accumulate(A, A + 1, 10, 1, 0) == _lib.FA_ERR_ALIGN
    assert fa.fa_accumulate(0, 0, 0, 1, 0) == _lib.FA_OK


def test_params_structs_match_the_header(tmp_path):
    """The ctypes mirrors of fa_fwd_params / fa_bwd_params have the C layout:
    a small C program built against include/fa.h prints every field's offset."""
    import shutil
    import subprocess
    if not shutil.which("gcc"):
        pytest.skip("gcc not available")
    fields = {"fa_fwd_params": _lib.FwdParams, "fa_bwd_params": _lib.BwdParams}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "fa.h"', "int main(void) {"]
    for cname, cls in fields.items():
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for f, _ in cls._fields_:
            lines.append(f'printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    lines.append("return 0; }")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    cuda_inc = "/usr/local/cuda/include"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, "-o", str(exe), str(src)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {tuple(l.split()[:2]): int(l.split()[2]) for l in out if l.strip()}
    for cname, cls in fields.items():
        assert got[(cname, "size")] == ctypes.sizeof(cls), cname
        for f, _ in cls._fields_:
            assert got[(cname, f)] == getattr(cls, f).offset, (cname, f)


def test_unified_entries_reject_bad_arguments(lib):
    assert _lib.load().fa_forward(None, None) == _lib.FA_ERR_NULL
    assert _lib.load().fa_backward(None, None) == _lib.FA_ERR_NULL
    base = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=1, Sq=128, Sk=128, D=128, scale=0.1, causal=0, dtype=1)
    assert fa.fa_forward(0, **base, dropout_p=-0.1) == _lib.FA_ERR_ARG
    assert fa.fa_forward(0, **base, dropout_p=1.0) == _lib.FA_ERR_ARG
    assert fa.fa_forward(0, **base, mask=A) == _lib.FA_ERR_NULL          # a mask needs its strides
    assert fa.fa_forward(0, **{**base, "D": 512}, dropout_p=0.1) == _lib.FA_ERR_HEADDIM
    assert fa.fa_forward(0, **{**base, "B": 0}, dropout_p=0.1) == _lib.FA_OK
    assert fa.fa_forward(0, **{**base, "B": 2}, q_stride=(7, 64, 64)) == _lib.FA_ERR_STRIDE
    bb = dict(q=A, k=A, v=A, o=A, dout=A, lse=A, dq=A, dk=A, dv=A, workspace=A, workspace_bytes=1 << 30, B=1, H=1,
              Sq=128, Sk=128, D=128, scale=0.1, causal=0, deterministic=0, dtype=1)
    assert fa.fa_backward(0, **bb, dropout_p=float("nan")) == _lib.FA_ERR_ARG
    assert fa.fa_backward(0, **{**bb, "D": 512}) == _lib.FA_ERR_HEADDIM
    assert fa.fa_backward(0, **{**bb, "B": 2, "H": 2}, dq_stride=(64, 0, 64)) == _lib.FA_ERR_STRIDE


def test_every_launch_reports_its_own_status():
    """Kernels launch through cudaLaunchKernelEx and the calls return that
    launch's status: no <<<>>> launch followed by a thread-global error query,
    which would also report an error that other code left pending."""
    import glob
    import os
    csrc = os.path.join(os.path.dirname(fa.__file__), "csrc")
    sources = glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cpp"))
    assert sources
    for path in sources:
        text = open(path).read()
        assert "<<<" not in text, path
        assert "cudaPeekAtLastError" not in text, path
        # the shared-memory limit is raised once per kernel and device, not per launch
        if not path.endswith("fa_api.cpp"):
            assert "cudaFuncSetAttribute" not in text, path


def test_forward_tiling_arguments_are_checked_before_any_device_work():
    """fa_forward's block_n / q_tiles: 0 (automatic), 64/128 and 1/2; a manual
    tiling takes D = 64/128 without mask or dropout (FA_ERR_ARG otherwise).
    All of these are found before a pointer is inspected."""
    from tiled_attention_18_b200 import _lib
    base = dict(q=16, k=16, v=16, o=16, lse=16, B=1, H=1, Sq=64, Sk=64, D=128, scale=0.1, causal=0, dtype=1)
    assert _lib.fa_forward(0, **base, block_n=96) == -10
    assert _lib.fa_forward(0, **base, q_tiles=3) == -10
    assert _lib.fa_forward(0, **base, q_tiles=-1) == -10
    assert _lib.fa_forward(0, **{**base, "D": 256}, block_n=64) == -10
    assert _lib.fa_forward(0, **base, block_n=64, dropout_p=0.1) == -10
    assert _lib.fa_forward(0, **base, q_tiles=1, mask=16, mask_stride=(0, 0, 64)) == -10

"""CPU tests of the C ABI: the library loads, exports every declared symbol,
and rejects bad arguments before making any CUDA call."""
from __future__ import annotations

import ctypes
import glob
import os
import re

import numpy as np
import pytest
import torch

from scaled_dot_product_10_b200 import attn
from scaled_dot_product_10_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return attn.load_library()


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?\w+[\s\*]+(attn_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_entry_points():
    names = declared_functions()
    assert "attn_fwd" in names and "attn_status" in names and "attn_strerror" in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(declared_functions()) <= set(attn.EXPORTED)


def test_every_bound_entry_point_is_declared():
    missing = sorted(set(attn.EXPORTED) - set(declared_functions()))
    assert not missing, f"bound but not declared in include/: {missing}"


def test_strerror(lib):
    for code in range(6):
        assert attn.attn_strerror(code)
    assert "unknown" in attn.attn_strerror(99)


# Fake device addresses: validation rejects the call before any CUDA use, so
# these are never dereferenced.
A = 0x10000


def call(lib, q=A, k=A, v=A, o=None, lse=None, b=1, hq=2, hkv=2, sq=256, sk=256, d=128,
         causal=0, scale=0.088):
    o = A if o is None else o
    lse = A if lse is None else lse
    return lib.attn_fwd(q, k, v, o, lse, b, hq, hkv, sq, sk, d, causal, scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), attn.ATTN_ERR_INVALID),
    (dict(k=0), attn.ATTN_ERR_INVALID),
    (dict(v=0), attn.ATTN_ERR_INVALID),
    (dict(o=0), attn.ATTN_ERR_INVALID),
    (dict(lse=0), attn.ATTN_ERR_INVALID),
    (dict(b=0), attn.ATTN_ERR_INVALID),
    (dict(hq=-1), attn.ATTN_ERR_INVALID),
    (dict(sk=0), attn.ATTN_ERR_INVALID),
    (dict(hq=6, hkv=4), attn.ATTN_ERR_INVALID),
    (dict(d=64), attn.ATTN_ERR_UNSUPPORTED),
    (dict(d=256), attn.ATTN_ERR_UNSUPPORTED),
    (dict(causal=1, sq=512, sk=256), attn.ATTN_ERR_UNSUPPORTED),
    (dict(causal=2), attn.ATTN_ERR_INVALID),
    (dict(scale=float("nan")), attn.ATTN_ERR_INVALID),
    (dict(scale=float("inf")), attn.ATTN_ERR_INVALID),
    (dict(q=A + 8), attn.ATTN_ERR_ALIGN),
    (dict(k=A + 4), attn.ATTN_ERR_ALIGN),
    (dict(v=A + 2), attn.ATTN_ERR_ALIGN),
    (dict(o=A + 8), attn.ATTN_ERR_ALIGN),
    (dict(lse=A + 2), attn.ATTN_ERR_ALIGN),
    (dict(b=1 << 20, hq=1 << 10, hkv=1 << 10, sq=1 << 20, sk=128), attn.ATTN_ERR_INVALID),
])
def test_validation_codes(lib, kw, code):
    assert call(lib, **kw) == code


def test_error_writes_nothing(lib):
    o = np.full(64, 7, dtype=np.uint16)
    lse = np.full(16, 3.0, dtype=np.float32)
    rc = call(lib, o=o.ctypes.data, lse=lse.ctypes.data, d=64)
    assert rc == attn.ATTN_ERR_UNSUPPORTED
    assert np.all(o == 7) and np.all(lse == 3.0)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_no_device_reports_cuda_error(lib):
    assert call(lib) == attn.ATTN_ERR_CUDA


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks validation on the no-device path")
@pytest.mark.parametrize("scale", [0.0, -0.0, -0.1, -3.0, 1e-30, 1e3])
def test_any_finite_scale_passes_validation(lib, scale):
    # Every finite scale is a valid argument (the formula has no sign or size
    # condition on it): validation accepts it and the call then fails only for
    # want of a device.
    assert call(lib, scale=scale) == attn.ATTN_ERR_CUDA
    assert call(lib, scale=scale, causal=1) == attn.ATTN_ERR_CUDA


def test_host_workspace_bytes(lib):
    b, hq, hkv, s = 2, 4, 2, 300
    q = b * s * hq * 128 * 2
    kv = b * s * hkv * 128 * 2
    l = b * hq * s * 4
    r = lambda x: (x + 255) // 256 * 256
    assert lib.attn_fwd_host_workspace_bytes(b, hq, hkv, s, s, 128) == 2 * r(q) + 2 * r(kv) + r(l)
    assert lib.attn_fwd_host_workspace_bytes(b, hq, hkv, s, s, 64) == 0
    assert lib.attn_fwd_host_workspace_bytes(b, 3, 2, s, s, 128) == 0


def test_host_entry_validation(lib):
    args = (A, A, A, A, A, 1, 2, 2, 256, 256, 128, 0, 0.088)
    need = lib.attn_fwd_host_workspace_bytes(1, 2, 2, 256, 256, 128)
    assert lib.attn_fwd_host(*args, None, need, None) == attn.ATTN_ERR_INVALID
    assert lib.attn_fwd_host(*args, A, need - 1, None) == attn.ATTN_ERR_INVALID
    assert lib.attn_fwd_host(*args, A + 16, need, None) == attn.ATTN_ERR_ALIGN


def test_split_workspace_bytes(lib):
    b, hq, s, n = 2, 4, 300, 5
    rows = b * hq * s
    r = lambda x: (x + 255) // 256 * 256
    assert lib.attn_fwd_split_workspace_bytes(b, hq, s, n) == r(n * rows * 128 * 4) + n * rows * 4
    assert lib.attn_fwd_split_workspace_bytes(b, hq, s, 0) == 0
    assert lib.attn_fwd_split_workspace_bytes(0, hq, s, 2) == 0


def test_split_entry_validation(lib):
    # 256 keys = 2 key blocks: 3 requested ranges become 2.
    args = (A, A, A, A, A, 1, 2, 2, 256, 256, 128, 0, 0.088)
    need2 = lib.attn_fwd_split_workspace_bytes(1, 2, 256, 2)
    assert lib.attn_fwd_split(*args, 0, A, need2, None) == attn.ATTN_ERR_INVALID
    assert lib.attn_fwd_split(*args, 2, None, need2, None) == attn.ATTN_ERR_INVALID
    assert lib.attn_fwd_split(*args, 2, A, need2 - 1, None) == attn.ATTN_ERR_INVALID
    assert lib.attn_fwd_split(*args, 3, A, need2 - 1, None) == attn.ATTN_ERR_INVALID
    assert lib.attn_fwd_split(*args, 2, A + 16, need2, None) == attn.ATTN_ERR_ALIGN
    # A workspace of exactly the documented size passes validation (the call
    # then fails only for want of a device, or runs if there is one).
    if not torch.cuda.is_available():
        assert lib.attn_fwd_split(*args, 2, A, need2, None) == attn.ATTN_ERR_CUDA
        assert lib.attn_fwd_split(*args, 3, A, need2, None) == attn.ATTN_ERR_CUDA
    bad = (A, A, A, A, A, 1, 2, 2, 256, 256, 64, 0, 0.088)
    assert lib.attn_fwd_split(*bad, 2, A, need2, None) == attn.ATTN_ERR_UNSUPPORTED
    causal_rect = (A, A, A, A, A, 1, 2, 2, 256, 128, 128, 1, 0.088)
    assert lib.attn_fwd_split(*causal_rect, 2, A, need2, None) == attn.ATTN_ERR_UNSUPPORTED


def test_partials_entry_validation(lib):
    ok = (A, A, A, A, A, 1, 2, 2, 256, 256, 128, 0, 0.088)
    f = lib.attn_fwd_partials
    assert f(A, A, A, 0, A, *ok[5:], None) == attn.ATTN_ERR_INVALID
    assert f(A, A, A, A, 0, *ok[5:], None) == attn.ATTN_ERR_INVALID
    assert f(A, A, A, A + 8, A, *ok[5:], None) == attn.ATTN_ERR_ALIGN
    assert f(*ok[:10], 64, 0, 0.088, None) == attn.ATTN_ERR_UNSUPPORTED


@pytest.mark.parametrize("kw,code", [
    (dict(op=0), attn.ATTN_ERR_INVALID),
    (dict(lp=0), attn.ATTN_ERR_INVALID),
    (dict(o=0), attn.ATTN_ERR_INVALID),
    (dict(lse=0), attn.ATTN_ERR_INVALID),
    (dict(n=0), attn.ATTN_ERR_INVALID),
    (dict(s=-1), attn.ATTN_ERR_INVALID),
    (dict(d=64), attn.ATTN_ERR_UNSUPPORTED),
    (dict(op=A + 4), attn.ATTN_ERR_ALIGN),
    (dict(o=A + 8), attn.ATTN_ERR_ALIGN),
    (dict(lse=A + 2), attn.ATTN_ERR_ALIGN),
])
def test_merge_validation_codes(lib, kw, code):
    a = dict(op=A, lp=A, n=2, b=1, h=2, s=256, d=128, o=A, lse=A)
    a.update(kw)
    assert lib.attn_merge_partials(a["op"], a["lp"], a["n"], a["b"], a["h"], a["s"], a["d"],
                                   a["o"], a["lse"], None) == code


def test_python_binding_rejects_wrong_dtype():
    q = torch.zeros(1, 8, 2, 128)
    with pytest.raises(TypeError):
        attn.attn_fwd(q, q, q)


def test_python_binding_requires_cuda_tensors():
    q = torch.zeros(1, 8, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        attn.attn_fwd(q, q, q)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(OSError):
        attn.load_library(str(tmp_path / "nope.so"))


def test_window_entry_validation(lib):
    f = lib.attn_fwd_window
    ok = (A, A, A, A, A, 1, 2, 2, 256, 256, 128)
    assert f(*ok, -1, 0.088, None) == attn.ATTN_ERR_INVALID
    assert f(*ok[:10], 64, 10, 0.088, None) == attn.ATTN_ERR_UNSUPPORTED
    assert f(A, A, A, A, A, 1, 2, 2, 512, 256, 128, 10, 0.088, None) == attn.ATTN_ERR_UNSUPPORTED
    assert f(A + 8, *ok[1:], 10, 0.088, None) == attn.ATTN_ERR_ALIGN
    if not torch.cuda.is_available():
        assert f(*ok, 10, 0.088, None) == attn.ATTN_ERR_CUDA


def test_varlen_entry_validation(lib):
    f = lib.attn_fwd_varlen
    # q, k, v, o, lse, cu_q, cu_k, batch, max_q, max_k, total_q, total_k, h_q, h_kv, d,
    # causal, window_left, scale
    ok = [A, A, A, A, A, A, A, 2, 300, 300, 400, 400, 4, 2, 128, 1, -1, 0.088, None]

    def call_with(**kw):
        names = ["q", "k", "v", "o", "lse", "cq", "ck", "b", "mq", "mk", "tq", "tk", "hq",
                 "hkv", "d", "causal", "w", "scale", "stream"]
        a = dict(zip(names, ok))
        a.update(kw)
        return f(*[a[n] for n in names])

    assert call_with(cq=0) == attn.ATTN_ERR_INVALID
    assert call_with(ck=0) == attn.ATTN_ERR_INVALID
    assert call_with(b=0) == attn.ATTN_ERR_INVALID
    assert call_with(mq=0) == attn.ATTN_ERR_INVALID
    assert call_with(tq=0) == attn.ATTN_ERR_INVALID
    assert call_with(hq=3) == attn.ATTN_ERR_INVALID
    assert call_with(d=64) == attn.ATTN_ERR_UNSUPPORTED
    assert call_with(causal=2) == attn.ATTN_ERR_INVALID
    assert call_with(w=-2) == attn.ATTN_ERR_INVALID
    assert call_with(causal=0, w=5) == attn.ATTN_ERR_INVALID
    assert call_with(cq=A + 2) == attn.ATTN_ERR_ALIGN
    assert call_with(q=A + 8) == attn.ATTN_ERR_ALIGN
    if not torch.cuda.is_available():
        assert call_with() == attn.ATTN_ERR_CUDA


def test_bwd_entry_validation(lib):
    f = lib.attn_bwd
    need = lib.attn_bwd_workspace_bytes(1, 2, 256)
    assert need == 2 * 1 * 2 * 256 * 4
    assert lib.attn_bwd_workspace_bytes(0, 2, 256) == 0
    base = [A, A, A, A, A, A, A, A, A, 1, 2, 2, 256, 256, 128, 1, -1, 0.088, A, need, None]

    def call_with(i, val):
        a = list(base)
        a[i] = val
        return f(*a)

    for i in range(9):          # any null pointer
        assert call_with(i, 0) == attn.ATTN_ERR_INVALID
    assert call_with(18, 0) == attn.ATTN_ERR_INVALID          # workspace
    assert call_with(19, need - 1) == attn.ATTN_ERR_INVALID   # too small
    assert call_with(18, A + 16) == attn.ATTN_ERR_ALIGN       # workspace alignment
    assert call_with(6, A + 8) == attn.ATTN_ERR_ALIGN         # dq
    assert call_with(14, 64) == attn.ATTN_ERR_UNSUPPORTED     # d
    assert call_with(16, -2) == attn.ATTN_ERR_INVALID         # window
    a = list(base)
    a[15], a[16] = 0, 5                                       # window without causal
    assert f(*a) == attn.ATTN_ERR_INVALID
    if not torch.cuda.is_available():
        assert f(*base) == attn.ATTN_ERR_CUDA


def test_fp8_entry_validation(lib):
    f = lib.attn_fwd_fp8
    ok = (A, A, A, A, A, 1, 2, 2, 256, 256, 128, 0, 0.088)
    assert f(*ok, float("nan"), 1.0, 1.0, None) == attn.ATTN_ERR_INVALID
    assert f(*ok, 1.0, float("inf"), 1.0, None) == attn.ATTN_ERR_INVALID
    assert f(*ok, 1.0, 1.0, float("nan"), None) == attn.ATTN_ERR_INVALID
    assert f(*ok[:10], 64, 0, 0.088, 1.0, 1.0, 1.0, None) == attn.ATTN_ERR_UNSUPPORTED
    assert f(A + 8, *ok[1:], 1.0, 1.0, 1.0, None) == attn.ATTN_ERR_ALIGN
    if not torch.cuda.is_available():
        assert f(*ok, 1.0, 1.0, 1.0, None) == attn.ATTN_ERR_CUDA


def test_wait_timeout_setter(lib):
    """Host-only: any bound is accepted and 0 restores the default."""
    assert lib.attn_set_wait_timeout_ns(5_000_000_000) == attn.ATTN_OK
    assert lib.attn_set_wait_timeout_ns(0) == attn.ATTN_OK
    attn.set_wait_timeout_ns(3_000_000_000)
    attn.set_wait_timeout_ns(0)
    with pytest.raises(ValueError):
        attn.set_wait_timeout_ns(-1)

"""CPU tests of the Python binding's argument marshalling (no GPU needed).

Every entry point of scaled_dot_product_10_b200.attn is called with CPU
tensors presented as CUDA tensors and a stand-in for the C library that
records what it is called with.  The tests check the exact argument list
each entry passes to its C function, matched by name to the parameters
include/*.h declares (pointers, sizes, flags, scale, stream handle), and the
binding's checks:
one device for every tensor of a call, a torch stream of that device, host
tensors for the host-buffer entry.
"""
from __future__ import annotations

import contextlib
import glob
import math
import os
import re
import types

import pytest
import torch

from scaled_dot_product_10_b200 import attn


class FakeCuda:
    """A CPU tensor presented as a tensor on CUDA device ``index``."""

    def __init__(self, t: torch.Tensor, index: int = 0):
        self._t = t
        self.device = torch.device("cuda", index)
        self.is_cuda = True

    def __getattr__(self, name):
        return getattr(self._t, name)


class FakeLib:
    """Records each C call as (name, args) and returns 0 (ATTN_OK), or the
    given value for size queries."""

    def __init__(self, sizes=None):
        self.calls = []
        self.sizes = sizes or {}

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            return self.sizes.get(name, 0)
        return fn


@pytest.fixture
def lib(monkeypatch):
    fake = FakeLib({"attn_bwd_workspace_bytes": 4096, "attn_fwd_split_workspace_bytes": 8192,
                    "attn_fwd_num_splits": 3})
    monkeypatch.setattr(attn, "load_library", lambda path=None: fake)
    monkeypatch.setattr(attn, "_on_device", lambda dev: contextlib.nullcontext())
    return fake


def bf16(*shape, index=0):
    return FakeCuda(torch.zeros(shape, dtype=torch.bfloat16), index)


def f32(*shape, index=0):
    return FakeCuda(torch.zeros(shape, dtype=torch.float32), index)


def u8(n, index=0):
    return FakeCuda(torch.zeros(n, dtype=torch.uint8), index)


B, SQ, SK, HQ, HKV, D = 2, 5, 7, 4, 2, 128
STREAM = 1234  # a raw stream handle is passed through unchanged


def qkv(index_k=0):
    return bf16(B, SQ, HQ, D), bf16(B, SK, HKV, D, index=index_k), bf16(B, SK, HKV, D)


_HEADERS = "".join(open(p).read() for p in sorted(
    glob.glob(os.path.join(os.path.dirname(__file__), "..", "include", "*.h"))))


def declared(name: str) -> list[str]:
    """Parameter names of C function ``name`` as include/*.h declares it."""
    m = re.search(r"^(?:int|size_t)\s+" + name + r"\s*\(([^;]*?)\)\s*;", _HEADERS,
                  re.S | re.M)
    assert m, f"{name} is not declared"
    return [re.split(r"[\s*]+", a.strip())[-1] for a in m.group(1).split(",")]


def last(lib, name):
    assert lib.calls and lib.calls[-1][0] == name, [c[0] for c in lib.calls]
    return lib.calls[-1][1]


def check_call(lib, name, **want):
    """The last C call was ``name`` with exactly these arguments, matched to
    the declaration's parameter names."""
    args = last(lib, name)
    params = declared(name)
    assert len(args) == len(params), f"{name}: {len(args)} arguments for {params}"
    assert dict(zip(params, args)) == want


def test_attn_fwd_arguments(lib):
    q, k, v = qkv()
    o, lse = bf16(B, SQ, HQ, D), f32(B, HQ, SQ)
    ro, rl = attn.attn_fwd(q, k, v, causal=True, scale=0.3, o=o, lse=lse, stream=STREAM)
    assert ro is o and rl is lse
    check_call(lib, "attn_fwd", q=q.data_ptr(), k=k.data_ptr(), v=v.data_ptr(), o=o.data_ptr(),
               lse=lse.data_ptr(), batch=B, h_q=HQ, h_kv=HKV, s_q=SQ, s_k=SK, d=D, causal=1,
               scale=0.3, stream=STREAM)


def test_attn_fwd_default_scale(lib):
    q, k, v = qkv()
    attn.attn_fwd(q, k, v, o=bf16(B, SQ, HQ, D), lse=f32(B, HQ, SQ), stream=STREAM)
    assert last(lib, "attn_fwd")[12] == pytest.approx(1 / math.sqrt(D))


def test_attn_fwd_window_arguments(lib):
    q, k, v = qkv()
    o, lse = bf16(B, SQ, HQ, D), f32(B, HQ, SQ)
    attn.attn_fwd_window(q, k, v, 3, scale=0.2, o=o, lse=lse, stream=STREAM)
    check_call(lib, "attn_fwd_window", q=q.data_ptr(), k=k.data_ptr(), v=v.data_ptr(),
               o=o.data_ptr(), lse=lse.data_ptr(), batch=B, h_q=HQ, h_kv=HKV, s_q=SQ, s_k=SK,
               d=D, window_left=3, scale=0.2, stream=STREAM)


def test_attn_fwd_varlen_arguments(lib):
    tq, tk = 9, 11
    q, k, v = bf16(tq, HQ, D), bf16(tk, HKV, D), bf16(tk, HKV, D)
    cu_q = FakeCuda(torch.tensor([0, 4, 9], dtype=torch.int32))
    cu_k = FakeCuda(torch.tensor([0, 5, 11], dtype=torch.int32))
    o, lse = bf16(tq, HQ, D), f32(HQ, tq)
    attn.attn_fwd_varlen(q, k, v, cu_q, cu_k, 5, 6, causal=True, scale=0.1, window_left=2,
                         o=o, lse=lse, stream=STREAM)
    check_call(lib, "attn_fwd_varlen", q=q.data_ptr(), k=k.data_ptr(), v=v.data_ptr(),
               o=o.data_ptr(), lse=lse.data_ptr(), cu_seqlens_q=cu_q.data_ptr(),
               cu_seqlens_k=cu_k.data_ptr(), batch=2, max_seqlen_q=5, max_seqlen_k=6,
               total_q=tq, total_k=tk, h_q=HQ, h_kv=HKV, d=D, causal=1, window_left=2,
               scale=0.1, stream=STREAM)


def test_attn_bwd_arguments(lib):
    q, k, v = qkv()
    o, dout, lse = bf16(B, SQ, HQ, D), bf16(B, SQ, HQ, D), f32(B, HQ, SQ)
    dq, dk, dv = bf16(B, SQ, HQ, D), bf16(B, SK, HKV, D), bf16(B, SK, HKV, D)
    ws = u8(4096)
    got = attn.attn_bwd(q, k, v, o, lse, dout, causal=True, scale=0.25, window_left=4, dq=dq,
                        dk=dk, dv=dv, workspace=ws, stream=STREAM)
    assert got == (dq, dk, dv)
    check_call(lib, "attn_bwd", q=q.data_ptr(), k=k.data_ptr(), v=v.data_ptr(), o=o.data_ptr(),
               dout=dout.data_ptr(), lse=lse.data_ptr(), dq=dq.data_ptr(), dk=dk.data_ptr(),
               dv=dv.data_ptr(), batch=B, h_q=HQ, h_kv=HKV, s_q=SQ, s_k=SK, d=D, causal=1,
               window_left=4, scale=0.25, workspace=ws.data_ptr(), workspace_bytes=4096,
               stream=STREAM)


def test_attn_bwd_checks_its_tensors(lib):
    q, k, v = qkv()
    o, dout, lse = bf16(B, SQ, HQ, D), bf16(B, SQ, HQ, D), f32(B, HQ, SQ)
    out = dict(dq=bf16(B, SQ, HQ, D), dk=bf16(B, SK, HKV, D), dv=bf16(B, SK, HKV, D),
               workspace=u8(4096), stream=STREAM)
    with pytest.raises(ValueError, match="dk must have shape"):
        attn.attn_bwd(q, k, v, o, lse, dout, **{**out, "dk": bf16(B, SQ, HKV, D)})
    with pytest.raises(ValueError, match="workspace"):
        attn.attn_bwd(q, k, v, o, lse, dout, **{**out, "workspace": u8(4096, index=1)})
    with pytest.raises(ValueError, match="dout must be on"):
        attn.attn_bwd(q, k, v, o, lse, bf16(B, SQ, HQ, D, index=1), **out)
    with pytest.raises(TypeError, match="lse must be"):
        attn.attn_bwd(q, k, v, o, bf16(B, HQ, SQ), dout, **out)
    assert not any(c[0] == "attn_bwd" for c in lib.calls)


def test_attn_fwd_fp8_arguments(lib):
    q = FakeCuda(torch.zeros(B, SQ, HQ, D, dtype=torch.float8_e4m3fn))
    k = FakeCuda(torch.zeros(B, SK, HKV, D, dtype=torch.float8_e4m3fn))
    v = FakeCuda(torch.zeros(B, SK, HKV, D, dtype=torch.float8_e4m3fn))
    o, lse = bf16(B, SQ, HQ, D), f32(B, HQ, SQ)
    attn.attn_fwd_fp8(q, k, v, 0.5, 0.25, 2.0, causal=False, scale=0.3, o=o, lse=lse,
                      stream=STREAM)
    check_call(lib, "attn_fwd_fp8", q=q.data_ptr(), k=k.data_ptr(), v=v.data_ptr(),
               o=o.data_ptr(), lse=lse.data_ptr(), batch=B, h_q=HQ, h_kv=HKV, s_q=SQ, s_k=SK,
               d=D, causal=0, scale=0.3, q_scale=0.5, k_scale=0.25, v_scale=2.0, stream=STREAM)


def test_attn_fwd_split_arguments(lib):
    q, k, v = qkv()
    o, lse, ws = bf16(B, SQ, HQ, D), f32(B, HQ, SQ), u8(8192)
    attn.attn_fwd_split(q, k, v, causal=False, scale=0.3, o=o, lse=lse, workspace=ws,
                        stream=STREAM)
    name, args = lib.calls[0]
    assert name == "attn_fwd_num_splits"
    assert dict(zip(declared(name), args)) == dict(batch=B, h_q=HQ, h_kv=HKV, s_q=SQ, s_k=SK,
                                                   d=D, causal=0)
    check_call(lib, "attn_fwd_split", q=q.data_ptr(), k=k.data_ptr(), v=v.data_ptr(),
               o=o.data_ptr(), lse=lse.data_ptr(), batch=B, h_q=HQ, h_kv=HKV, s_q=SQ, s_k=SK,
               d=D, causal=0, scale=0.3, num_splits=3, workspace=ws.data_ptr(),
               workspace_bytes=8192, stream=STREAM)


def test_attn_fwd_partials_arguments(lib):
    q, k, v = qkv()
    op, lp = f32(B, HQ, SQ, D), f32(B, HQ, SQ)
    attn.attn_fwd_partials(q, k, v, causal=True, scale=0.3, o_part=op, lse_part=lp,
                           stream=STREAM)
    check_call(lib, "attn_fwd_partials", q=q.data_ptr(), k=k.data_ptr(), v=v.data_ptr(),
               o_part=op.data_ptr(), lse_part=lp.data_ptr(), batch=B, h_q=HQ, h_kv=HKV, s_q=SQ,
               s_k=SK, d=D, causal=1, scale=0.3, stream=STREAM)
    attn.attn_fwd_partials_shard(q, k, v, causal=True, scale=0.3, o_part=op, lse_part=lp,
                                 stream=STREAM)
    # default diagonal: the whole-problem mask, s_k - s_q
    check_call(lib, "attn_fwd_partials_shard", q=q.data_ptr(), k=k.data_ptr(), v=v.data_ptr(),
               o_part=op.data_ptr(), lse_part=lp.data_ptr(), batch=B, h_q=HQ, h_kv=HKV,
               s_q=SQ, s_k=SK, d=D, causal=1, diag_offset=SK - SQ, scale=0.3, stream=STREAM)


def test_merge_partials_arguments(lib):
    n = 3
    op, lp = f32(n, B, HQ, SQ, D), f32(n, B, HQ, SQ)
    o, lse = bf16(B, SQ, HQ, D), f32(B, HQ, SQ)
    attn.merge_partials(op, lp, o=o, lse=lse, stream=STREAM)
    check_call(lib, "attn_merge_partials", o_parts=op.data_ptr(), lse_parts=lp.data_ptr(),
               n_parts=n, batch=B, h_q=HQ, s_q=SQ, d=D, o=o.data_ptr(), lse=lse.data_ptr(),
               stream=STREAM)
    with pytest.raises(ValueError, match="lse_parts is on"):
        attn.merge_partials(op, f32(n, B, HQ, SQ, index=1), o=o, lse=lse, stream=STREAM)


def test_host_entry_arguments(lib):
    q = torch.zeros(B, SQ, HQ, D, dtype=torch.bfloat16)
    k = torch.zeros(B, SK, HKV, D, dtype=torch.bfloat16)
    v = torch.zeros(B, SK, HKV, D, dtype=torch.bfloat16)
    o = torch.zeros(B, SQ, HQ, D, dtype=torch.bfloat16)
    lse = torch.zeros(B, HQ, SQ, dtype=torch.float32)
    ws = u8(1000)
    attn.attn_fwd_host(q, k, v, o, lse, ws, causal=True, scale=0.3, stream=STREAM)
    check_call(lib, "attn_fwd_host", q=q.data_ptr(), k=k.data_ptr(), v=v.data_ptr(),
               o=o.data_ptr(), lse=lse.data_ptr(), batch=B, h_q=HQ, h_kv=HKV, s_q=SQ, s_k=SK,
               d=D, causal=1, scale=0.3, workspace=ws.data_ptr(), workspace_bytes=1000,
               stream=STREAM)
    with pytest.raises(ValueError, match="host tensor"):
        attn.attn_fwd_host(FakeCuda(q), k, v, o, lse, ws, stream=STREAM)
    with pytest.raises(ValueError, match="workspace must be a CUDA tensor"):
        attn.attn_fwd_host(q, k, v, o, lse, torch.zeros(1000, dtype=torch.uint8), stream=STREAM)


@pytest.mark.parametrize("entry", ["attn_fwd", "attn_fwd_window", "attn_fwd_split",
                                   "attn_fwd_partials", "attn_fwd_partials_shard"])
def test_inputs_on_two_devices_are_refused(lib, entry):
    q, k, v = qkv(index_k=1)
    args = (q, k, v, 2) if entry == "attn_fwd_window" else (q, k, v)
    with pytest.raises(ValueError, match="k is on cuda:1"):
        getattr(attn, entry)(*args, stream=STREAM)
    assert lib.calls == []


def test_stream_of_another_device_is_refused(lib):
    q, k, v = qkv()
    other = types.SimpleNamespace(device=torch.device("cuda", 1), cuda_stream=99)
    with pytest.raises(ValueError, match="stream belongs to cuda:1"):
        attn.attn_fwd(q, k, v, o=bf16(B, SQ, HQ, D), lse=f32(B, HQ, SQ), stream=other)
    same = types.SimpleNamespace(device=torch.device("cuda", 0), cuda_stream=99)
    attn.attn_fwd(q, k, v, o=bf16(B, SQ, HQ, D), lse=f32(B, HQ, SQ), stream=same)
    assert last(lib, "attn_fwd")[-1] == 99


def test_cpu_inputs_are_refused(lib):
    q, k, v = qkv()
    with pytest.raises(ValueError, match="v must be a CUDA tensor"):
        attn.attn_fwd(q, k, v._t, stream=STREAM)
    assert lib.calls == []

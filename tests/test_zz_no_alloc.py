"""The allocation-free host entry point (attn_fwd_host_static).

Some callers cannot allocate device memory at call time -- a plugin that is
handed only host arrays by an application owning all device memory, or code
that cannot afford the synchronisation cudaMalloc/cudaFree may imply.  For
them the library stages the copies in its own static device array.  This
checks, through the C ABI, that two calls in a row give the same result as
the workspace-taking entry point (attn_fwd_host) and as the FP64 oracle,
within the parity tolerances, and that oversized problems are refused.  Collected last so a
stop-at-first-failure run has already run every other test.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from parity import assert_within, gather_rows, metrics
from scaled_dot_product_10_b200 import attn
from scaled_dot_product_10_b200.workloads import make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


def _pinned(b, hq, hkv, s, seed):
    q, k, v = make_qkv(b, hq, hkv, s, s, seed=seed)
    q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    o = torch.empty_like(q).pin_memory()
    lse = torch.empty((b, hq, s), dtype=torch.float32).pin_memory()
    return q, k, v, o, lse


def _static_call(q, k, v, o, lse, causal):
    lib = attn.load_library()
    b, s, hq, d = q.shape
    hkv = k.shape[2]
    stream = torch.cuda.current_stream()
    rc = lib.attn_fwd_host_static(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  lse.data_ptr(), b, hq, hkv, s, s, d, int(causal),
                                  1.0 / math.sqrt(d), stream.cuda_stream)
    assert rc == attn.ATTN_OK, attn.attn_strerror(rc)
    assert lib.attn_status(stream.cuda_stream) == attn.ATTN_OK


def _workspace_call(q, k, v, causal):
    b, s, hq, d = q.shape
    hkv = k.shape[2]
    o = torch.empty_like(q).pin_memory()
    lse = torch.empty((b, hq, s), dtype=torch.float32).pin_memory()
    ws = torch.empty(attn.host_workspace_bytes(b, hq, hkv, s, s), dtype=torch.uint8, device="cuda")
    attn.attn_fwd_host(q, k, v, o, lse, ws, causal=causal, scale=1.0 / math.sqrt(d))
    assert attn.attn_status() == attn.ATTN_OK
    return o, lse


def test_static_entry_matches_workspace_entry_twice():
    # Two calls in a row through the shared staging array (different sizes,
    # so the second overwrites part of what the first left there); each
    # result is then compared with the workspace-taking entry point and with
    # the FP64 oracle, within the parity tolerances.
    cases = [((2, 4, 2, 513, 7100), True), ((1, 8, 1, 1000, 7101), False)]
    runs = []
    for (b, hq, hkv, s, seed), causal in cases:
        q, k, v, o, lse = _pinned(b, hq, hkv, s, seed)
        _static_call(q, k, v, o, lse, causal)
        runs.append((q, k, v, o, lse, causal))
    for q, k, v, o, lse, causal in runs:
        b, s = q.shape[0], q.shape[1]
        o_ws, lse_ws = _workspace_call(q, k, v, causal)
        a, la = gather_rows(o, lse, None)
        r, lr = gather_rows(o_ws, lse_ws, None)
        assert_within(metrics(a, la, r, lr), f"static vs workspace b={b} s={s}")
        o_ref, l_ref, _ = oracle.attn_fwd(q, k, v, causal, 1.0 / math.sqrt(q.shape[3]))
        assert_within(metrics(a, la, o_ref, l_ref), f"static vs oracle b={b} s={s}")


def test_static_entry_refuses_oversized_problem():
    lib = attn.load_library()
    # 16 heads x 8192 rows x 128 x 2 B = 32 MiB for q alone: over the limit.
    need = lib.attn_fwd_host_workspace_bytes(1, 16, 16, 8192, 8192, 128)
    assert need > attn.STATIC_STAGING_BYTES
    a = 0x10000
    rc = lib.attn_fwd_host_static(a, a, a, a, a, 1, 16, 16, 8192, 8192, 128, 0, 0.088, None)
    assert rc == attn.ATTN_ERR_TOO_LARGE
    assert "static" in attn.attn_strerror(rc)

"""Property tests of the C ABI's argument validation (CPU, no device).

include/attn_fwd.h and include/attn_bwd.h state which arguments each entry
rejects and with which code, before any CUDA call.  On a machine without a
GPU a call that passes validation reaches its first CUDA call and returns
ATTN_ERR_CUDA, so every call here returns either the documented error code
or ATTN_ERR_CUDA.  Hypothesis draws valid calls and calls with exactly one
violated rule (derandomized, so every run checks the same draws).

Device pointers are fake addresses that are never dereferenced: the module
is skipped wherever a CUDA device is visible, so no call can launch.
"""
from __future__ import annotations

import math

import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

from scaled_dot_product_10_b200 import attn

pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="fake device addresses: runs only without a device")
SETTINGS = dict(deadline=None, derandomize=True, database=None, max_examples=150)
A = 0x10000  # 256-byte aligned fake address
OK_VALIDATION = attn.ATTN_ERR_CUDA  # passed validation, then found no device


@pytest.fixture(scope="module")
def lib():
    return attn.load_library()


@st.composite
def valid_sizes(draw):
    h_kv = draw(st.integers(1, 8))
    h_q = h_kv * draw(st.integers(1, 8))
    b = draw(st.integers(1, 16))
    s_k = draw(st.integers(1, 1 << 15))
    causal = draw(st.integers(0, 1))
    s_q = draw(st.integers(1, s_k)) if causal else draw(st.integers(1, 1 << 15))
    scale = draw(st.sampled_from([0.088, 0.0, -0.0, -1.5, 1e-30, 1e3]))
    return dict(b=b, h_q=h_q, h_kv=h_kv, s_q=s_q, s_k=s_k, d=128, causal=causal, scale=scale)


# One violated rule: (name, change to the arguments, expected code).
VIOLATIONS = {
    "null q": (lambda a: a.update(q=0), attn.ATTN_ERR_INVALID),
    "null o": (lambda a: a.update(o=0), attn.ATTN_ERR_INVALID),
    "null lse": (lambda a: a.update(lse=0), attn.ATTN_ERR_INVALID),
    "batch 0": (lambda a: a.update(b=0), attn.ATTN_ERR_INVALID),
    "negative s_q": (lambda a: a.update(s_q=-a["s_q"]), attn.ATTN_ERR_INVALID),
    "s_k 0": (lambda a: a.update(s_k=0, causal=0), attn.ATTN_ERR_INVALID),
    "h_q not a multiple of h_kv": (lambda a: a.update(h_kv=a["h_q"] + 1), attn.ATTN_ERR_INVALID),
    "NaN scale": (lambda a: a.update(scale=math.nan), attn.ATTN_ERR_INVALID),
    "infinite scale": (lambda a: a.update(scale=-math.inf), attn.ATTN_ERR_INVALID),
    "causal 2": (lambda a: a.update(causal=2), attn.ATTN_ERR_INVALID),
    "d 64": (lambda a: a.update(d=64), attn.ATTN_ERR_UNSUPPORTED),
    "causal with s_q > s_k": (lambda a: a.update(causal=1, s_q=a["s_k"] + 1),
                              attn.ATTN_ERR_UNSUPPORTED),
    "q misaligned": (lambda a: a.update(q=A + 8), attn.ATTN_ERR_ALIGN),
    "o misaligned": (lambda a: a.update(o=A + 2), attn.ATTN_ERR_ALIGN),
    "lse misaligned": (lambda a: a.update(lse=A + 2), attn.ATTN_ERR_ALIGN),
}


def fwd(lib, a):
    return lib.attn_fwd(a.get("q", A), A, A, a.get("o", A), a.get("lse", A), a["b"], a["h_q"],
                        a["h_kv"], a["s_q"], a["s_k"], a["d"], a["causal"], a["scale"], None)


@settings(**SETTINGS)
@given(valid_sizes(), st.sampled_from([None] + sorted(VIOLATIONS)))
def test_attn_fwd_codes(lib, a, violation):
    want = OK_VALIDATION
    if violation is not None:
        change, want = VIOLATIONS[violation]
        change(a)
    assert fwd(lib, a) == want, (violation, a)


@settings(**SETTINGS)
@given(valid_sizes(), st.integers(-3, 1 << 16),
       st.sampled_from([None, "null q", "d 64", "q misaligned", "batch 0"]))
def test_attn_fwd_window_codes(lib, a, window, violation):
    """The window entry is causal: s_q <= s_k; window_left < 0 is invalid."""
    a["causal"] = 1
    a["s_q"] = min(a["s_q"], a["s_k"])
    want = OK_VALIDATION if window >= 0 else attn.ATTN_ERR_INVALID
    if violation is not None:
        change, code = VIOLATIONS[violation]
        change(a)
        if window >= 0:
            want = code
        elif code == attn.ATTN_ERR_ALIGN or code == attn.ATTN_ERR_UNSUPPORTED:
            want = None  # two violations: either code is a correct answer
    got = lib.attn_fwd_window(a.get("q", A), A, A, A, A, a["b"], a["h_q"], a["h_kv"], a["s_q"],
                              a["s_k"], a["d"], window, a["scale"], None)
    if want is None:
        assert got in (attn.ATTN_ERR_INVALID, code), (violation, window, a)
    else:
        assert got == want, (violation, window, a)


@settings(**SETTINGS)
@given(valid_sizes(), st.integers(-1, 300), st.sampled_from(
    [None, "null dout", "null dk", "window without causal", "window below -1",
     "small workspace", "workspace misaligned", "dv misaligned"] + sorted(VIOLATIONS)))
def test_attn_bwd_codes(lib, a, window, violation):
    ws_need = int(lib.attn_bwd_workspace_bytes(a["b"], a["h_q"], a["s_q"]))
    args = dict(q=A, dout=A, dk=A, dv=A, ws=A, ws_bytes=ws_need)
    if window >= 0:
        a["causal"] = 1
        a["s_q"] = min(a["s_q"], a["s_k"])
        args["ws_bytes"] = int(lib.attn_bwd_workspace_bytes(a["b"], a["h_q"], a["s_q"]))
    want = OK_VALIDATION
    extra = {
        "null dout": (lambda: args.update(dout=0), attn.ATTN_ERR_INVALID),
        "null dk": (lambda: args.update(dk=0), attn.ATTN_ERR_INVALID),
        "window without causal": (lambda: a.update(causal=0), attn.ATTN_ERR_INVALID),
        "window below -1": (lambda: None, attn.ATTN_ERR_INVALID),
        "small workspace": (lambda: args.update(ws_bytes=args["ws_bytes"] - 1),
                            attn.ATTN_ERR_INVALID),
        "workspace misaligned": (lambda: args.update(ws=A + 16), attn.ATTN_ERR_ALIGN),
        "dv misaligned": (lambda: args.update(dv=A + 8), attn.ATTN_ERR_ALIGN),
    }
    w = window
    if violation in extra:
        change, want = extra[violation]
        change()
        if violation == "window below -1":
            w = -2
        if violation == "window without causal" and window < 0:
            want = OK_VALIDATION  # no window: non-causal is fine
    elif violation is not None:
        change, want = VIOLATIONS[violation]
        change(a)
        if violation in ("null o", "null lse", "o misaligned", "lse misaligned"):
            args.update(o=a.pop("o", A), lse=a.pop("lse", A))
        if violation in ("causal 2", "s_k 0", "causal with s_q > s_k") and window >= 0:
            return  # these change the mask a window needs: covered by the forward test
    if violation == "small workspace" and args["ws_bytes"] < 0:
        return
    got = lib.attn_bwd(a.get("q", args["q"]), A, A, args.get("o", A), args["dout"],
                       args.get("lse", A), A, args["dk"], args["dv"], a["b"], a["h_q"],
                       a["h_kv"], a["s_q"], a["s_k"], a["d"], a["causal"], w, a["scale"],
                       args["ws"], max(0, args["ws_bytes"]), None)
    assert got == want, (violation, window, a, args)

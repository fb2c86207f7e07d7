"""GPU parity of the backward (dQ, dK, dV) against the FP64 oracle's
backward, on the same seeded BF16 inputs and incoming gradient dO.

The GPU backward starts from the GPU forward's O (BF16) and LSE (FP32) and
rounds P^T and dS to BF16 before their tensor-core products; dQ, dK, dV are
FP32 sums rounded to BF16.  An emulation of exactly those rounding points in
FP32 (every other step exact) lands at relative L2 errors of 2.3e-3 to
2.7e-3 and largest errors of 2.4e-3 to 5.4e-3 of the largest gradient
against the FP64 oracle on the shapes below; the bar is about four times
that: relative L2 <= 1e-2 and max |d| <= 2e-2 * max |ref| for each of dQ,
dK, dV.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from scaled_dot_product_10_b200 import attn
from scaled_dot_product_10_b200.workloads import make_qkv

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)
REL_L2 = 1e-2
MAX_REL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    attn.load_library()
    torch.cuda.set_device(0)


def run_bwd(q, k, v, dout, causal, scale=SCALE, window_left=-1):
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    if window_left >= 0:
        o, lse = attn.attn_fwd_window(qd, kd, vd, window_left, scale=scale)
    else:
        o, lse = attn.attn_fwd(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = attn.attn_bwd(qd, kd, vd, o, lse, dod, causal=causal or window_left >= 0,
                               scale=scale, window_left=window_left)
    rc = attn.attn_status()
    assert rc == attn.ATTN_OK, attn.attn_strerror(rc)
    return dq, dk, dv


def check_bwd(q, k, v, dout, causal, scale=SCALE, window_left=-1, what=""):
    got = run_bwd(q, k, v, dout, causal, scale, window_left)
    ref = oracle.attn_bwd(q, k, v, dout, causal or window_left >= 0, scale,
                          window_left=window_left)
    out = {}
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        g = g.float().cpu().double().numpy()
        assert np.all(np.isfinite(g)), f"{what}: {name} not finite"
        rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300)
        mx = np.max(np.abs(g - r)) / max(np.max(np.abs(r)), 1e-300)
        out[name] = (rel, mx)
        assert rel <= REL_L2, f"{what}: {name} relative L2 {rel:.3e}"
        assert mx <= MAX_REL, f"{what}: {name} max error {mx:.3e} of max |ref|"
    return out


def grads_in(b, hq, hkv, s_q, s_k, seed):
    q, k, v = make_qkv(b, hq, hkv, s_q, s_k, seed=seed)
    dout = make_qkv(b, hq, hkv, s_q, s_k, seed=seed + 1)[0]
    return q, k, v, dout


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_tiny(causal):
    check_bwd(*grads_in(1, 2, 2, 256, 256, 11000), causal, what=f"tiny causal={causal}")


@pytest.mark.parametrize("s", [1, 63, 64, 65, 127, 129, 200, 383, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_tails(s, causal):
    check_bwd(*grads_in(1, 2, 2, s, s, 11100 + s), causal, what=f"s={s} causal={causal}")


@pytest.mark.parametrize("h_q,h_kv", [(16, 2), (16, 1), (6, 3), (8, 8)])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_head_sharing(h_q, h_kv, causal):
    check_bwd(*grads_in(2, h_q, h_kv, 384, 384, 11200 + h_kv), causal,
              what=f"h {h_q}/{h_kv} causal={causal}")


@pytest.mark.parametrize("s_q,s_k", [(100, 1000), (1, 300), (300, 700), (640, 643)])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_rectangular(s_q, s_k, causal):
    check_bwd(*grads_in(1, 4, 2, s_q, s_k, 11300 + s_q), causal,
              what=f"{s_q}x{s_k} causal={causal}")


@pytest.mark.parametrize("s_q,s_k", [(700, 300), (1000, 129)])
def test_bwd_more_queries_than_keys(s_q, s_k):
    # Without a mask s_q > s_k is allowed: more query blocks than key blocks,
    # a ragged last key block (keys past s_k get no weight in dQ).
    check_bwd(*grads_in(2, 4, 2, s_q, s_k, 11350 + s_q), False, what=f"{s_q}x{s_k}")


@pytest.mark.parametrize("w", [1, 100, 255])
def test_bwd_window(w):
    check_bwd(*grads_in(1, 4, 4, 1000, 1000, 11400 + w), True, window_left=w, what=f"w={w}")


def test_bwd_window_zero_gives_zero_dq_dk():
    # Each row sees only its diagonal key: P = 1, so dS = dP - D = 0 and
    # dQ = dK = 0 exactly (a relative error is meaningless there); dV = dO
    # row for row.  The GPU's rounding residual must stay tiny in absolute
    # terms (inputs are O(1)).
    q, k, v, dout = grads_in(1, 4, 4, 1000, 1000, 11450)
    dq, dk, dv = run_bwd(q, k, v, dout, True, window_left=0)
    assert torch.max(torch.abs(dq.float())) <= 1e-3
    assert torch.max(torch.abs(dk.float())) <= 1e-3
    _, _, dv_ref = oracle.attn_bwd(q, k, v, dout, True, SCALE, window_left=0)
    g = dv.float().cpu().double().numpy()
    assert np.max(np.abs(g - dv_ref)) <= MAX_REL * np.max(np.abs(dv_ref))


@pytest.mark.parametrize("b,h_q,h_kv,s_q,s_k,w", [
    (2, 4, 2, 128, 384, 0),     # two whole key blocks before the first window
    (2, 4, 2, 100, 700, 37),    # unseen keys end inside a block
    (1, 4, 4, 200, 1000, 130),
    (8, 8, 4, 128, 1100, 3),    # more key-block items than SMs
])
def test_bwd_window_keys_no_query_sees(b, h_q, h_kv, s_q, s_k, w):
    """Bottom-right window with s_q < s_k: keys before the first query's
    window (j < s_k - s_q - w) get no weight, so their dK and dV are exactly
    zero, and whole key blocks of them have no work item of their own.  The
    outputs start as NaN so that a row nobody wrote shows."""
    q, k, v, dout = grads_in(b, h_q, h_kv, s_q, s_k, 11460 + s_q + w)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = attn.attn_fwd_window(qd, kd, vd, w, scale=SCALE)
    dq, dk, dv = (torch.full_like(t, float("nan")) for t in (qd, kd, vd))
    attn.attn_bwd(qd, kd, vd, o, lse, dod, causal=True, scale=SCALE, window_left=w, dq=dq,
                  dk=dk, dv=dv)
    rc = attn.attn_status()
    assert rc == attn.ATTN_OK, attn.attn_strerror(rc)
    unseen = s_k - s_q - w
    assert torch.all(dk[:, :unseen] == 0) and torch.all(dv[:, :unseen] == 0)
    ref = oracle.attn_bwd(q, k, v, dout, True, SCALE, window_left=w)
    for name, g, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref):
        g = g.float().cpu().double().numpy()
        assert np.all(np.isfinite(g)), f"{name} not finite (a row left unwritten)"
        if w == 0 and name != "dV":
            # one visible key per row: dQ = dK = 0 exactly (see above)
            assert np.max(np.abs(g)) <= 1e-3
            continue
        rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300)
        mx = np.max(np.abs(g - r)) / max(np.max(np.abs(r)), 1e-300)
        assert rel <= REL_L2, f"{name} relative L2 {rel:.3e}"
        assert mx <= MAX_REL, f"{name} max error {mx:.3e} of max |ref|"


@pytest.mark.parametrize("scale", [-0.09, 0.0, 0.5])
def test_bwd_scales(scale):
    check_bwd(*grads_in(1, 2, 2, 512, 512, 11500), True, scale=scale, what=f"scale={scale}")


def test_bwd_many_items_more_than_sms():
    check_bwd(*grads_in(2, 8, 4, 1536, 1536, 11600), True, what="persistent")


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_gqa_workload_shape(causal):
    # The GQA workload's shape (16 query heads on 2 key/value heads, 2048
    # rows) at batch 2.
    check_bwd(*grads_in(2, 16, 2, 2048, 2048, 11700), causal, what=f"gqa 2048 causal={causal}")


def test_bwd_deterministic():
    q, k, v, dout = grads_in(2, 8, 2, 1000, 1000, 11800)
    a = run_bwd(q, k, v, dout, True)
    b = run_bwd(q, k, v, dout, True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)

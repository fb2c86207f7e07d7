"""Shared helpers for the GPU-vs-oracle parity tests.

Tolerances (the stated bar for this path): max |dO| <= 2e-2, relative L2 of
O <= 5e-3, max |dLSE| <= 1e-3, all against the FP64 oracle on identical
BF16 inputs.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from scaled_dot_product_10_b200 import attn

MAX_ABS_O = 2e-2
REL_L2_O = 5e-3
MAX_ABS_LSE = 1e-3


def run_gpu(q, k, v, causal, scale):
    """Run the CUDA path on CPU BF16 tensors; returns (o, lse) CUDA tensors."""
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = attn.attn_fwd(qd, kd, vd, causal=causal, scale=scale)
    rc = attn.attn_status()
    assert rc == attn.ATTN_OK, attn.attn_strerror(rc)
    return o, lse


def gather_rows(o_gpu, lse_gpu, rows):
    """o_gpu [b, s, h, d], lse_gpu [b, h, s] -> o [b, h, n, d], lse [b, h, n] (float64)."""
    o = o_gpu.float().cpu()
    l = lse_gpu.float().cpu()
    b, s, h, d = o.shape
    if rows is None:
        return o.permute(0, 2, 1, 3).double().numpy(), l.double().numpy()
    r = torch.as_tensor(rows, dtype=torch.long)  # [b, h, n]
    bi = torch.arange(b)[:, None, None].expand_as(r)
    hi = torch.arange(h)[None, :, None].expand_as(r)
    return o[bi, r, hi].double().numpy(), l[bi, hi, r].double().numpy()


def metrics(o, lse, o_ref, lse_ref):
    d = o - o_ref
    return {
        "max_abs_o": float(np.max(np.abs(d))),
        "rel_l2_o": float(np.linalg.norm(d) / max(np.linalg.norm(o_ref), 1e-300)),
        "max_abs_lse": float(np.max(np.abs(lse - lse_ref))),
    }


def assert_within(m, what=""):
    assert np.isfinite(m["max_abs_o"]) and np.isfinite(m["max_abs_lse"]), f"{what}: non-finite {m}"
    assert m["max_abs_o"] <= MAX_ABS_O, f"{what}: max|dO| {m}"
    assert m["rel_l2_o"] <= REL_L2_O, f"{what}: rel-L2 {m}"
    assert m["max_abs_lse"] <= MAX_ABS_LSE, f"{what}: max|dLSE| {m}"


def check(q, k, v, causal, scale, rows=None, what=""):
    o_gpu, lse_gpu = run_gpu(q, k, v, causal, scale)
    o_ref, lse_ref, _ = oracle.attn_fwd(q, k, v, causal, scale, rows=rows)
    o, lse = gather_rows(o_gpu, lse_gpu, rows)
    m = metrics(o, lse, o_ref, lse_ref)
    assert_within(m, what)
    return m

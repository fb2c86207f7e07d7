"""GPU parity of the FP8 (E4M3) forward against the FP64 oracle on the same
E4M3 inputs and per-tensor scales.

The oracle evaluates the definition on the exact dequantized inputs.  The
kernel's products Q K^T and P V are exact FP8 products accumulated in FP32;
its one coarse rounding is the weights P, stored as E4M3 (3 mantissa bits,
as 2^6 P).  Bars:
- relative L2 of O <= 5e-2: an FP32 emulation of that rounding point alone
  gives 1.9e-2 to 2.6e-2 on N(0, 1) inputs of these shapes (7e-3 when K is
  drawn x8), so the bar is twice the worst;
- max |dO| <= 2^-4 max|V| + 1e-2: O is a convex combination of V rows and
  round-to-nearest E4M3 moves each normal weight by at most 2^-4 of itself,
  so the weights' rounding moves O by at most 2^-4 max|V|; 1e-2 covers
  subnormal weights and the BF16 rounding of O (the emulation's largest
  error is 4.7e-2 for N(0, 1) inputs and 6.3e-2 with K x8, against bounds
  of about 0.3);
- |dLSE| <= 1e-3: LSE comes from the FP32 sums of the unrounded weights and
  keeps the BF16 bar.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from parity import gather_rows
from scaled_dot_product_10_b200 import attn
from scaled_dot_product_10_b200.workloads import WORKLOADS, make_qkv_fp8, sample_rows

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)
REL_L2 = 5e-2
MAX_ABS_LSE = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    attn.load_library()
    torch.cuda.set_device(0)


def check_fp8(b, hq, hkv, s_q, s_k, causal, seed, scale=SCALE, rows=None, k_scale=1.0):
    q8, k8, v8, qs, ks, vs = make_qkv_fp8(b, hq, hkv, s_q, s_k, seed=seed, k_scale=k_scale)
    o, lse = attn.attn_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), qs, ks, vs, causal=causal,
                               scale=scale)
    rc = attn.attn_status()
    assert rc == attn.ATTN_OK, attn.attn_strerror(rc)
    o_ref, l_ref = oracle.attn_fwd_fp8(q8, k8, v8, qs, ks, vs, causal, scale, rows=rows)
    oo, ll = gather_rows(o, lse, rows)
    d = oo - o_ref
    rel = np.linalg.norm(d) / np.linalg.norm(o_ref)
    max_abs_o = 2.0 ** -4 * float(v8.float().abs().max()) * vs + 1e-2
    assert np.all(np.isfinite(oo)) and np.all(np.isfinite(ll))
    assert rel <= REL_L2, f"rel-L2 {rel:.3e}"
    assert np.max(np.abs(d)) <= max_abs_o, f"max |dO| {np.max(np.abs(d)):.3e} > {max_abs_o:.3e}"
    assert np.max(np.abs(ll - l_ref)) <= MAX_ABS_LSE, f"max |dLSE| {np.max(np.abs(ll - l_ref)):.3e}"
    return rel


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_tiny(causal):
    check_fp8(1, 2, 2, 256, 256, causal, 12000)


@pytest.mark.parametrize("s", [1, 64, 127, 129, 383, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_tails(s, causal):
    check_fp8(1, 2, 2, s, s, causal, 12100 + s)


@pytest.mark.parametrize("h_q,h_kv", [(16, 2), (16, 1), (6, 3)])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_head_sharing(h_q, h_kv, causal):
    check_fp8(2, h_q, h_kv, 384, 384, causal, 12200 + h_kv)


@pytest.mark.parametrize("s_q,s_k", [(100, 1000), (1, 4096), (300, 700)])
def test_fp8_causal_rectangular(s_q, s_k):
    check_fp8(1, 4, 2, s_q, s_k, True, 12300 + s_q)


@pytest.mark.parametrize("scale", [-0.09, 0.0, 0.3])
def test_fp8_scales(scale):
    check_fp8(1, 2, 2, 512, 512, True, 12400, scale=scale)


def test_fp8_sharp_softmax_rescale():
    # K drawn x8 before quantisation: the row maximum keeps growing past the
    # FP8 path's 2^2 rescale threshold.
    check_fp8(1, 2, 2, 1024, 1024, True, 12500, k_scale=8.0)


@pytest.mark.parametrize("name", ["mha_b8_h16_s4096", "mha_b1_h16_s32768_k3",
                                  "gqa_b8_h16_kv2_s2048"])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_workload_shapes(name, causal):
    w = WORKLOADS[name]
    rows = sample_rows(w.batch, w.h_q, w.seq, 64, seed=w.seed + 12600)
    check_fp8(w.batch, w.h_q, w.h_kv, w.seq, w.seq, causal, w.seed, rows=rows,
              k_scale=w.k_scale)


def test_fp8_deterministic():
    q8, k8, v8, qs, ks, vs = make_qkv_fp8(2, 4, 2, 1000, 1000, seed=12700)
    a = attn.attn_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), qs, ks, vs, causal=True)
    b = attn.attn_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), qs, ks, vs, causal=True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])

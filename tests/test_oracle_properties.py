"""Property tests of the FP64 oracle over many small random shapes (CPU).

The pins check chosen cases; here Hypothesis draws batch, head grouping
(MHA, GQA, MQA), s_q <= s_k or any s_k without the causal mask, head dims,
causal with and without a sliding window, and positive or negative scales.
Each draw compares the oracle with independent library routines on the same
inputs:

* forward: torch's float64 scaled_dot_product_attention with the explicit
  boolean mask (key j visible to query i iff j <= i + s_k - s_q, and with a
  window of W also j >= i + s_k - s_q - W), and scipy's logsumexp of the
  masked scaled scores for LSE;
* backward: torch's float64 autograd of the same SDPA for L = sum(O * dO);
* FP8 forward: arbitrary E4M3 codes with per-tensor scales, decoded by
  torch's float8_e4m3fn conversion, then the forward check above.

The draws are derandomized, so every run checks the same examples.
"""
from __future__ import annotations

import numpy as np
import pytest
import scipy.special
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from scaled_dot_product_10_b200.workloads import make_qkv

SETTINGS = dict(deadline=None, derandomize=True, database=None,
                suppress_health_check=[HealthCheck.too_slow])


@st.composite
def problems(draw):
    b = draw(st.integers(1, 2))
    h_kv = draw(st.integers(1, 3))
    h_q = h_kv * draw(st.integers(1, 3))
    d = draw(st.sampled_from([4, 8, 16, 32]))
    causal = draw(st.booleans())
    s_q = draw(st.integers(1, 24))
    s_k = draw(st.integers(s_q, s_q + 16)) if causal else draw(st.integers(1, 40))
    window = draw(st.sampled_from([-1, 0, 1, 3, 7])) if causal else -1
    scale = draw(st.sampled_from([0.05, 0.3, 1.0, -0.4]))
    seed = draw(st.integers(0, 10_000))
    return b, h_q, h_kv, s_q, s_k, d, causal, window, scale, seed


def visible(s_q, s_k, causal, window):
    """[s_q, s_k] boolean: key j is visible to query i."""
    i = torch.arange(s_q)[:, None]
    j = torch.arange(s_k)[None, :]
    allow = torch.ones(s_q, s_k, dtype=torch.bool)
    if causal:
        allow &= j <= i + (s_k - s_q)
        if window >= 0:
            allow &= j >= i + (s_k - s_q) - window
    return allow


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@settings(max_examples=60, **SETTINGS)
@given(problems())
def test_forward_matches_torch_sdpa_and_scipy_logsumexp(lib, prob):
    b, h_q, h_kv, s_q, s_k, d, causal, window, scale, seed = prob
    q, k, v = make_qkv(b, h_q, h_kv, s_q, s_k, seed=seed, d=d)
    mask = visible(s_q, s_k, causal, window)
    qt = q.double().transpose(1, 2)                                   # [b, h_q, s_q, d]
    kt = k.double().transpose(1, 2).repeat_interleave(h_q // h_kv, dim=1)
    vt = v.double().transpose(1, 2).repeat_interleave(h_q // h_kv, dim=1)
    want = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask,
                                                            scale=scale).numpy()
    scores = (qt @ kt.transpose(-1, -2)) * scale
    want_lse = scipy.special.logsumexp(scores.masked_fill(~mask, float("-inf")).numpy(), axis=-1)
    o, lse, _ = oracle.attn_fwd(q, k, v, causal, scale, lib=lib, window_left=window)
    assert np.max(np.abs(o - want)) < 1e-10, prob
    assert np.max(np.abs(lse - want_lse)) < 1e-10, prob


@settings(max_examples=40, **SETTINGS)
@given(problems())
def test_backward_matches_torch_autograd(lib, prob):
    b, h_q, h_kv, s_q, s_k, d, causal, window, scale, seed = prob
    q, k, v = make_qkv(b, h_q, h_kv, s_q, s_k, seed=seed, d=d)
    dout = make_qkv(b, h_q, h_kv, s_q, s_k, seed=seed + 1, d=d)[0]
    mask = visible(s_q, s_k, causal, window)
    qt = q.double().transpose(1, 2).requires_grad_()
    kt = k.double().transpose(1, 2).requires_grad_()
    vt = v.double().transpose(1, 2).requires_grad_()
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale,
                                                         enable_gqa=True)
    (o * dout.double().transpose(1, 2)).sum().backward()
    want = [t.grad.transpose(1, 2).numpy() for t in (qt, kt, vt)]
    got = oracle.attn_bwd(q, k, v, dout, causal, scale, window_left=window, lib=lib)
    for name, g, w in zip(("dQ", "dK", "dV"), got, want):
        assert np.max(np.abs(g - w)) < 1e-10, (name, prob)


@st.composite
def fp8_problems(draw):
    b, h_q, h_kv, s_q, s_k, d, causal, window, scale, seed = draw(problems())
    # arbitrary E4M3 bit patterns, uniform over the 254 codes that are not
    # NaN (0x7f, 0xff): every exponent, subnormals and both zeros
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)
    n = b * s_q * h_q * d + 2 * b * s_k * h_kv * d
    bits = np.random.default_rng(seed).choice(codes, size=n)
    scales = [draw(st.sampled_from([2.0 ** -6, 0.01, 1.0 / 448, 0.5])) for _ in range(3)]
    return b, h_q, h_kv, s_q, s_k, d, causal, window, scale, bits, scales


@settings(max_examples=30, **SETTINGS)
@given(fp8_problems())
def test_fp8_forward_matches_torch_float8_decode_and_sdpa(lib, prob):
    """FP8 inputs stand for scale x E4M3 value: decoded by torch's own
    float8_e4m3fn conversion, scaled, then torch's float64 SDPA."""
    b, h_q, h_kv, s_q, s_k, d, causal, window, scale, bits, (sq8, sk8, sv8) = prob
    n_q, n_kv = b * s_q * h_q * d, b * s_k * h_kv * d
    raw = torch.from_numpy(bits)
    q8 = raw[:n_q].view(torch.float8_e4m3fn).reshape(b, s_q, h_q, d)
    k8 = raw[n_q:n_q + n_kv].view(torch.float8_e4m3fn).reshape(b, s_k, h_kv, d)
    v8 = raw[n_q + n_kv:].view(torch.float8_e4m3fn).reshape(b, s_k, h_kv, d)
    mask = visible(s_q, s_k, causal, window)
    qt = (q8.double() * sq8).transpose(1, 2)
    kt = (k8.double() * sk8).transpose(1, 2).repeat_interleave(h_q // h_kv, dim=1)
    vt = (v8.double() * sv8).transpose(1, 2).repeat_interleave(h_q // h_kv, dim=1)
    want = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask,
                                                            scale=scale).numpy()
    scores = (qt @ kt.transpose(-1, -2)) * scale
    want_lse = scipy.special.logsumexp(scores.masked_fill(~mask, float("-inf")).numpy(), axis=-1)
    o, lse = oracle.attn_fwd_fp8(q8, k8, v8, sq8, sk8, sv8, causal, scale, lib=lib,
                                 window_left=window)
    assert np.max(np.abs(o - want)) < 1e-9 * max(1.0, np.max(np.abs(want))), prob[:9]
    assert np.max(np.abs(lse - want_lse)) < 1e-9 * max(1.0, np.max(np.abs(want_lse))), prob[:9]

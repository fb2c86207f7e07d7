"""CPU tests of the seeded workloads: the metric's FLOP and byte counts, and
the input recipe both the CUDA path and the oracle are fed from."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from scaled_dot_product_10_b200.workloads import (EDGE_ROWS, HEAD_DIM, WORKLOADS, make_qkv,
                                                  make_qkv_fp8, sample_rows, workload_qkv)


def visible_pairs(s: int, causal: bool) -> int:
    """(query, key) pairs the mask leaves, counted one by one."""
    return sum((i + 1) if causal else s for i in range(s))


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_flops_are_four_d_per_visible_pair(name):
    """Q K^T and P V are 2 d FLOP each per (query, key) pair.  Non-causal
    counts every pair; causal takes half of them, the usual convention,
    which differs from the exact count s (s + 1) / 2 by a factor 1 + 1/s."""
    w = WORKLOADS[name]
    per_head = 4 * HEAD_DIM * w.batch * w.h_q
    assert w.flops(False) == per_head * visible_pairs(w.seq, False)
    exact = per_head * visible_pairs(w.seq, True)
    assert w.flops(True) == pytest.approx(exact / (1 + 1 / w.seq), rel=1e-12)


def test_headline_workload_counts():
    w = WORKLOADS["mha_b1_h16_s32768_k3"]
    assert w.flops(False) == 8.796093022208e12
    assert w.flops(True) == 4.398046511104e12
    # Q, K, V read once, O written once (BF16), LSE written once (FP32)
    assert w.algorithmic_bytes() == 538_968_064
    assert w.input_bytes() == 402_653_184  # above the 126 MB L2: no flush needed


@pytest.mark.parametrize("name", sorted(n for n, w in WORKLOADS.items() if w.seq <= 4096))
def test_byte_counts_match_the_tensors(name):
    """(The formula is the same for the larger workloads; their tensors are
    not drawn here.)"""
    w = WORKLOADS[name]
    q, k, v = workload_qkv(w)
    size = lambda t: t.numel() * t.element_size()  # noqa: E731
    assert w.input_bytes() == size(q) + size(k) + size(v)
    assert w.algorithmic_bytes() == 2 * size(q) + size(k) + size(v) + w.batch * w.h_q * w.seq * 4


def test_workload_table():
    seeds = [w.seed for w in WORKLOADS.values()]
    assert len(set(seeds)) == len(seeds)
    for w in WORKLOADS.values():
        assert w.h_q % w.h_kv == 0
        assert w.scale == pytest.approx(HEAD_DIM ** -0.5)
        assert w.sampled == (w.seq >= 8192)
    assert WORKLOADS["mha_b1_h16_s32768_k3"].k_scale == 3.0


def test_draws_are_deterministic_and_ordered():
    a = make_qkv(2, 4, 2, 33, 47, seed=5, d=16)
    b = make_qkv(2, 4, 2, 33, 47, seed=5, d=16)
    c = make_qkv(2, 4, 2, 33, 47, seed=6, d=16)
    for x, y, z in zip(a, b, c):
        assert x.dtype == torch.bfloat16
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
        assert not torch.equal(x, z)
    q, k, v = a
    assert q.shape == (2, 33, 4, 16) and k.shape == v.shape == (2, 47, 2, 16)
    # Q, K, V come from one generator in that order
    g = torch.Generator().manual_seed(5)
    want_q = torch.randn((2, 33, 4, 16), generator=g).to(torch.bfloat16)
    want_k = torch.randn((2, 47, 2, 16), generator=g).to(torch.bfloat16)
    assert torch.equal(q, want_q) and torch.equal(k, want_k)


def test_k_scale_touches_only_k():
    q1, k1, v1 = make_qkv(1, 2, 2, 20, 20, seed=9, d=8)
    q3, k3, v3 = make_qkv(1, 2, 2, 20, 20, seed=9, d=8, k_scale=3.0)
    assert torch.equal(q1, q3) and torch.equal(v1, v3)
    g = torch.Generator().manual_seed(9)
    torch.randn((1, 20, 2, 8), generator=g)
    want = (torch.randn((1, 20, 2, 8), generator=g) * 3.0).to(torch.bfloat16)
    assert torch.equal(k3, want)


def test_sample_rows_keeps_edges_and_is_seeded():
    r = sample_rows(2, 3, 1000, 40, seed=11)
    assert r.shape == (2, 3, 40) and r.dtype == np.int32
    for row in r.reshape(-1, 40):
        assert np.all(np.diff(row) > 0) and row[0] >= 0 and row[-1] < 1000
        assert set(EDGE_ROWS) | {999} <= set(row.tolist())
    assert np.array_equal(r, sample_rows(2, 3, 1000, 40, seed=11))
    assert not np.array_equal(r, sample_rows(2, 3, 1000, 40, seed=12))
    # asking for every row (or more) gives every row
    assert np.array_equal(sample_rows(1, 1, 50, 80, seed=1)[0, 0], np.arange(50))
    # short sequences keep the edges that exist
    assert sample_rows(1, 1, 3, 2, seed=1)[0, 0].tolist() == [0, 1, 2]


def test_fp8_inputs_use_the_full_e4m3_range():
    q8, k8, v8, sq, sk, sv = make_qkv_fp8(2, 4, 2, 40, 40, seed=21, d=32)
    g = torch.Generator().manual_seed(21)
    ref = [torch.randn(s, generator=g) for s in ((2, 40, 4, 32), (2, 40, 2, 32), (2, 40, 2, 32))]
    for x8, sc, x in zip((q8, k8, v8), (sq, sk, sv), ref):
        assert x8.dtype == torch.float8_e4m3fn
        assert sc == pytest.approx(float(x.abs().max()) / 448.0, rel=1e-7)
        deq = x8.float() * sc
        assert float(x8.float().abs().max()) == 448.0  # the largest entry maps to E4M3's max
        # E4M3 keeps 3 mantissa bits: normal values within 2^-4 relative
        big = x.abs() > 2.0 ** -6 * sc * 8
        assert torch.all((deq[big] - x[big]).abs() <= 2.0 ** -4 * x[big].abs())

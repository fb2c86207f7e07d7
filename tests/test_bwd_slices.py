"""The row-slice assembly of the oracle's backward (tests/bwd_slices.py)
equals the oracle's backward of the whole problem: every query row's
gradient contributions are its own, so the two differ only by the order of
FP64 additions in dK and dV.  Square and rectangular causal, non-causal,
GQA groups, ragged last slices."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bwd_slices import oracle_group
from scaled_dot_product_10_b200.workloads import make_qkv


@pytest.mark.parametrize("b,h_q,h_kv,s_q,s_k,causal,rows", [
    (2, 4, 2, 300, 300, True, 64),
    (2, 4, 2, 300, 300, False, 64),
    (1, 3, 1, 100, 257, True, 32),
    (1, 2, 2, 129, 129, True, 128),
    (1, 2, 1, 70, 70, False, 128),
])
def test_slices_equal_whole_oracle(b, h_q, h_kv, s_q, s_k, causal, rows):
    q, k, v = make_qkv(b, h_q, h_kv, s_q, s_k, seed=12000 + s_q + s_k)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(s_q)).to(torch.bfloat16)
    scale = 0.09
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, causal, scale)
    group = h_q // h_kv
    for bb in range(b):
        for g in range(h_kv):
            sq, sk, sv = oracle_group(q, k, v, dout, bb, g, group, causal, scale, rows=rows)
            np.testing.assert_allclose(sq, dq[bb, :, g * group:(g + 1) * group], rtol=0, atol=1e-12)
            np.testing.assert_allclose(sk, dk[bb, :, g], rtol=0, atol=1e-12)
            np.testing.assert_allclose(sv, dv[bb, :, g], rtol=0, atol=1e-12)

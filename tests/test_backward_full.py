"""GPU parity of the backward at the full sizes the benchmark times.

For each backward workload of bench.py (MHA batch 8 x 16 heads x 4096, MHA
4 x 16 x 8192, GQA 8 x 16/2 x 2048), both masks, the GPU forward and
backward run on the whole problem in the benchmark's launch configuration;
then one whole (batch, key/value head) group -- every query head of the
group, every row of dQ, every key row of dK and dV -- is compared with the
FP64 oracle.

The oracle's backward of a group is assembled from calls on slices of 128
query rows (tests/bwd_slices.py, which tests/test_bwd_slices.py checks
against whole-problem oracle calls on the CPU).

Tolerances: the same derived bars as tests/test_backward.py (relative L2
<= 1e-2 and max |d| <= 2e-2 * max |ref| per tensor): the GPU rounds P^T and
dS to BF16 and accumulates in FP32; neither error grows with the sequence
length.  dO is a seeded N(0, 1) draw made on the host.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from bwd_slices import oracle_group
from scaled_dot_product_10_b200 import attn
from scaled_dot_product_10_b200.workloads import WORKLOADS, workload_qkv

pytestmark = pytest.mark.gpu
REL_L2 = 1e-2
MAX_REL = 2e-2
# (workload, causal, sampled batch, sampled key/value head)
CASES = [
    ("mha_b8_h16_s4096", False, 7, 15),
    ("mha_b8_h16_s4096", True, 0, 0),
    ("mha_b4_h16_s8192", False, 3, 15),
    ("mha_b4_h16_s8192", True, 1, 7),
    ("gqa_b8_h16_kv2_s2048", False, 7, 1),
    ("gqa_b8_h16_kv2_s2048", True, 0, 0),
]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    attn.load_library()
    torch.cuda.set_device(0)


@pytest.mark.parametrize("name,causal,b,g", CASES)
def test_bwd_full_size_group(name, causal, b, g):
    w = WORKLOADS[name]
    q, k, v = workload_qkv(w)
    gen = torch.Generator().manual_seed(w.seed + 50)
    dout = torch.randn(q.shape, generator=gen).to(torch.bfloat16)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    o, lse = attn.attn_fwd(qd, kd, vd, causal=causal, scale=w.scale)
    dq, dk, dv = attn.attn_bwd(qd, kd, vd, o, lse, dod, causal=causal, scale=w.scale)
    rc = attn.attn_status()
    assert rc == attn.ATTN_OK, attn.attn_strerror(rc)
    group = w.h_q // w.h_kv
    hs = slice(g * group, (g + 1) * group)
    got = (dq[b, :, hs].float().cpu().double().numpy(),
           dk[b, :, g].float().cpu().double().numpy(),
           dv[b, :, g].float().cpu().double().numpy())
    del qd, kd, vd, dod, o, lse, dq, dk, dv
    ref = oracle_group(q, k, v, dout, b, g, group, causal, w.scale)
    for label, x, r in zip(("dQ", "dK", "dV"), got, ref):
        assert np.all(np.isfinite(x)), f"{name} causal={causal}: {label} not finite"
        rel = np.linalg.norm(x - r) / max(np.linalg.norm(r), 1e-300)
        mx = np.max(np.abs(x - r)) / max(np.max(np.abs(r)), 1e-300)
        assert rel <= REL_L2, f"{name} causal={causal} (b={b}, g={g}): {label} relative L2 {rel:.3e}"
        assert mx <= MAX_REL, f"{name} causal={causal} (b={b}, g={g}): {label} max {mx:.3e} of max |ref|"

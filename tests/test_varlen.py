"""GPU parity of the packed variable-length forward against the FP64
oracle (each sequence its own attention problem), and its bit-identity with
one attn_fwd call per sequence."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from parity import assert_within, metrics
from scaled_dot_product_10_b200 import attn
from scaled_dot_product_10_b200.workloads import make_qkv

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    attn.load_library()
    torch.cuda.set_device(0)


def packed(lens_q, lens_k, h_q, h_kv, seed):
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    q, k, v = make_qkv(1, h_q, h_kv, int(cu_q[-1]), int(cu_k[-1]), seed=seed)
    return q[0].contiguous(), k[0].contiguous(), v[0].contiguous(), cu_q, cu_k


def run_varlen(q, k, v, cu_q, cu_k, causal, window_left=-1, scale=SCALE):
    lq = np.diff(cu_q)
    lk = np.diff(cu_k)
    o, lse = attn.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cu_q).cuda(),
                                  torch.from_numpy(cu_k).cuda(), int(max(lq.max(), 1)),
                                  int(max(lk.max(), 1)), causal=causal, scale=scale,
                                  window_left=window_left)
    rc = attn.attn_status()
    assert rc == attn.ATTN_OK, attn.attn_strerror(rc)
    return o, lse


def check_varlen(lens_q, lens_k, h_q, h_kv, causal, seed, window_left=-1):
    q, k, v, cu_q, cu_k = packed(lens_q, lens_k, h_q, h_kv, seed)
    o, lse = run_varlen(q, k, v, cu_q, cu_k, causal, window_left)
    o_ref, l_ref = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, causal, SCALE,
                                          window_left=window_left)
    m = metrics(o.float().cpu().double().numpy(), lse.cpu().double().numpy(), o_ref, l_ref)
    assert_within(m, f"varlen {lens_q}/{lens_k} causal={causal} w={window_left}")
    return o, lse, (q, k, v, cu_q, cu_k)


MIXES = [
    [1, 127, 128, 129, 300, 1000],   # tile edges and a single row
    [2048, 17, 640, 5, 900],         # long and short mixed
    [256] * 6,                       # equal lengths (dense-like)
    [4000, 96],
]


@pytest.mark.parametrize("lens", MIXES)
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_matches_oracle(lens, causal):
    check_varlen(lens, lens, 4, 2, causal, seed=9500 + len(lens))


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_fewer_queries_than_keys(causal):
    # Per-sequence bottom-right mask: each sequence's queries are its last s_q.
    check_varlen([1, 100, 128, 333], [1, 700, 129, 2000], 8, 8, causal, seed=9600)


def test_varlen_empty_query_sequence():
    # A sequence with keys but no query rows contributes nothing.
    check_varlen([200, 0, 300], [200, 50, 300], 2, 1, False, seed=9650)


@pytest.mark.parametrize("h_q,h_kv", [(16, 2), (16, 1)])
def test_varlen_head_sharing(h_q, h_kv):
    check_varlen([500, 1200, 64], [500, 1200, 64], h_q, h_kv, True, seed=9700 + h_kv)


@pytest.mark.parametrize("w", [0, 100, 255])
def test_varlen_with_window(w):
    check_varlen([1000, 300, 129, 2000], [1000, 300, 129, 2000], 4, 4, True, seed=9750 + w,
                 window_left=w)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_is_bit_identical_to_one_call_per_sequence(causal):
    lens = [300, 1000, 129, 640]
    q, k, v, cu_q, cu_k = packed(lens, lens, 4, 2, 9800)
    o, lse = run_varlen(q, k, v, cu_q, cu_k, causal)
    for b in range(len(lens)):
        a, e = cu_q[b], cu_q[b + 1]
        ob, lb = attn.attn_fwd(q[None, a:e].contiguous().cuda(), k[None, a:e].contiguous().cuda(),
                               v[None, a:e].contiguous().cuda(), causal=causal, scale=SCALE)
        assert torch.equal(o[a:e], ob[0]), f"sequence {b} O"
        assert torch.equal(lse[:, a:e], lb[0]), f"sequence {b} LSE"


def test_varlen_outputs_stay_in_bounds():
    lens = [129, 1, 300]
    q, k, v, cu_q, cu_k = packed(lens, lens, 2, 2, 9900)
    total, h = int(cu_q[-1]), 2
    pad = 4096
    o_buf = torch.full((2 * pad + total * h * 128,), 77.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((2 * pad + h * total,), -5.0, dtype=torch.float32, device="cuda")
    o = o_buf[pad:pad + total * h * 128].view(total, h, 128)
    lse = l_buf[pad:pad + h * total].view(h, total)
    attn.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cu_q).cuda(),
                         torch.from_numpy(cu_k).cuda(), 300, 300, causal=True, scale=SCALE,
                         o=o, lse=lse)
    assert attn.attn_status() == attn.ATTN_OK
    assert torch.all(o_buf[:pad] == 77.0) and torch.all(o_buf[-pad:] == 77.0)
    assert torch.all(l_buf[:pad] == -5.0) and torch.all(l_buf[-pad:] == -5.0)
    o_ref, l_ref = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, True, SCALE)
    assert_within(metrics(o.float().cpu().double().numpy(), lse.cpu().double().numpy(), o_ref,
                          l_ref), "varlen guarded")


def test_varlen_many_sequences_more_items_than_sms():
    rng = np.random.default_rng(9950)
    lens = [int(x) for x in rng.integers(1, 1500, size=40)]
    check_varlen(lens, lens, 8, 2, True, seed=9951)

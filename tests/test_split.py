"""GPU parity of the split-KV forward and of the partial merge against the
FP64 oracle.

The merge (LSE = log sum_r exp LSE_r, O = sum_r exp(LSE_r - LSE) O_r) is the
online-softmax "local attention, then global reduction" of the rkmt.cn GPU
attention operator page, section 3.1.1, over whole key ranges; its result is
the plain attention of the whole key set, so the oracle of the unsplit
problem is the reference for every split count.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from parity import assert_within, gather_rows, metrics, run_gpu
from scaled_dot_product_10_b200 import attn
from scaled_dot_product_10_b200.workloads import make_qkv, sample_rows

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    attn.load_library()
    torch.cuda.set_device(0)


def run_split(q, k, v, causal, n_splits):
    o, lse = attn.attn_fwd_split(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=SCALE,
                                 n_splits=n_splits)
    rc = attn.attn_status()
    assert rc == attn.ATTN_OK, attn.attn_strerror(rc)
    return o, lse


@pytest.mark.parametrize("b,hq,hkv,sq,sk,causal,n", [
    (1, 4, 4, 300, 5000, False, 3),      # ragged query and key tails
    (1, 16, 16, 256, 32768, False, None),  # few queries, long keys: the library's count
    (2, 8, 2, 1000, 1000, True, 4),      # causal GQA: early rows see only the first ranges
    (1, 2, 2, 129, 129, True, 2),        # causal, second range = one key
    (1, 4, 1, 640, 640, True, 7),        # MQA; 7 requested, 5 key blocks -> 5 ranges
    (2, 4, 4, 64, 4096, False, 32),      # one key block per range
    (1, 2, 2, 1, 300, False, 3),         # a single query row
    (3, 6, 3, 200, 2000, False, 2),
    (1, 16, 16, 64, 32768, True, None),  # causal decode-like: bottom-right mask
    (2, 8, 2, 1, 8192, True, 5),         # one query row, causal
    (1, 4, 4, 300, 5000, True, 3),       # causal, ranges that early rows cannot see
    (1, 4, 4, 200, 300, True, 3),        # offset 100 inside the first key block
])
def test_split_matches_oracle(b, hq, hkv, sq, sk, causal, n):
    q, k, v = make_qkv(b, hq, hkv, sq, sk, seed=7100 + sq + sk)
    o, lse = run_split(q, k, v, causal, n)
    rows = None if b * hq * sq <= 8192 else sample_rows(b, hq, sq, 64, seed=7200 + sq)
    o_ref, l_ref, _ = oracle.attn_fwd(q, k, v, causal, SCALE, rows=rows)
    oo, ll = gather_rows(o, lse, rows)
    assert_within(metrics(oo, ll, o_ref, l_ref), f"split b{b} h{hq}/{hkv} {sq}x{sk} n={n}")


@pytest.mark.parametrize("causal", [False, True])
def test_one_range_is_bit_exact_with_attn_fwd(causal):
    q, k, v = make_qkv(2, 4, 2, 700, 700, seed=7300)
    o1, l1 = run_gpu(q, k, v, causal, SCALE)
    o2, l2 = run_split(q, k, v, causal, 1)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_split_is_deterministic_and_status_clean():
    q, k, v = make_qkv(1, 8, 8, 512, 8192, seed=7400)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o0, l0 = attn.attn_fwd_split(qd, kd, vd, scale=SCALE, n_splits=6)
    ws = torch.empty(attn.split_workspace_bytes(1, 8, 512, 6), dtype=torch.uint8, device="cuda")
    o, lse = torch.empty_like(o0), torch.empty_like(l0)
    for _ in range(50):
        attn.attn_fwd_split(qd, kd, vd, scale=SCALE, n_splits=6, o=o, lse=lse, workspace=ws)
    assert attn.attn_status() == attn.ATTN_OK
    assert torch.equal(o, o0) and torch.equal(lse, l0)
    assert attn.last_launch_count() == 2


def test_library_split_count():
    # Few pairs over long keys: several ranges; a workload that fills the
    # SMs: one.
    n = attn.num_splits(1, 16, 16, 256, 32768)
    assert 2 <= n <= 256
    assert attn.num_splits(8, 16, 16, 4096, 4096) == 1


def _oracle_partials(q, k, v, bounds):
    """Per-key-range oracle results: O_r (normalised over the range) and LSE_r."""
    o_parts, l_parts = [], []
    for lo, hi in bounds:
        o_r, l_r, _ = oracle.attn_fwd(q, k[:, lo:hi].contiguous(), v[:, lo:hi].contiguous(),
                                      False, SCALE)
        o_parts.append(o_r)  # [b, h, s, d]
        l_parts.append(l_r)  # [b, h, s]
    return np.stack(o_parts), np.stack(l_parts)


def test_merge_partials_of_oracle_ranges():
    # Partials computed by the oracle on three uneven key ranges merge into
    # the oracle's whole-sequence result.
    b, hq, hkv, sq, sk = 2, 4, 2, 96, 700
    q, k, v = make_qkv(b, hq, hkv, sq, sk, seed=7500)
    o_p, l_p = _oracle_partials(q, k, v, [(0, 100), (100, 450), (450, 700)])
    o, lse = attn.merge_partials(torch.from_numpy(o_p).float().cuda().contiguous(),
                                 torch.from_numpy(l_p).float().cuda().contiguous())
    assert attn.attn_status() == attn.ATTN_OK
    o_ref, l_ref, _ = oracle.attn_fwd(q, k, v, False, SCALE)
    oo, ll = gather_rows(o, lse, None)
    assert_within(metrics(oo, ll, o_ref, l_ref), "merge of oracle partials")


def test_merge_skips_empty_parts():
    # A part with LSE = -inf carries no weight and its O is never read (NaN
    # there must not leak); a row whose parts are all empty gives O = 0 and
    # LSE = -inf.
    b, hq, hkv, sq, sk = 1, 2, 2, 64, 300
    q, k, v = make_qkv(b, hq, hkv, sq, sk, seed=7600)
    o_p, l_p = _oracle_partials(q, k, v, [(0, 150), (150, 300)])
    o_p = np.concatenate([o_p, np.full_like(o_p[:1], np.nan)])
    l_p = np.concatenate([l_p, np.full_like(l_p[:1], -np.inf)])
    o, lse = attn.merge_partials(torch.from_numpy(o_p).float().cuda().contiguous(),
                                 torch.from_numpy(l_p).float().cuda().contiguous())
    o_ref, l_ref, _ = oracle.attn_fwd(q, k, v, False, SCALE)
    oo, ll = gather_rows(o, lse, None)
    assert_within(metrics(oo, ll, o_ref, l_ref), "merge with an empty part")
    empty_o = torch.full((1, 1, 2, 8, 128), float("nan"), device="cuda")
    empty_l = torch.full((1, 1, 2, 8), float("-inf"), device="cuda")
    o2, l2 = attn.merge_partials(empty_o, empty_l)
    assert torch.all(o2 == 0) and torch.all(torch.isneginf(l2))


def test_partials_of_key_shards_merge_to_the_whole():
    # The context-parallel data flow on one device: each key shard's
    # unmerged partial, gathered, merged.
    b, hq, hkv, sq, sk = 2, 8, 2, 384, 3000
    q, k, v = make_qkv(b, hq, hkv, sq, sk, seed=7700)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    cuts = [0, 1000, 1900, 3000]  # uneven shards, ragged key tails
    parts = [attn.attn_fwd_partials(qd, kd[:, lo:hi].contiguous(), vd[:, lo:hi].contiguous(),
                                    scale=SCALE) for lo, hi in zip(cuts[:-1], cuts[1:])]
    o_parts = torch.stack([p[0] for p in parts]).contiguous()
    l_parts = torch.stack([p[1] for p in parts]).contiguous()
    o, lse = attn.merge_partials(o_parts, l_parts)
    assert attn.attn_status() == attn.ATTN_OK
    rows = sample_rows(b, hq, sq, 64, seed=7701)
    o_ref, l_ref, _ = oracle.attn_fwd(q, k, v, False, SCALE, rows=rows)
    oo, ll = gather_rows(o, lse, rows)
    assert_within(metrics(oo, ll, o_ref, l_ref), "merged key shards")
    # Each partial alone is the oracle of its own shard.
    lo, hi = cuts[1], cuts[2]
    o_r, l_r, _ = oracle.attn_fwd(q, k[:, lo:hi].contiguous(), v[:, lo:hi].contiguous(), False,
                                  SCALE, rows=rows)
    r = torch.as_tensor(rows, dtype=torch.long)
    bi = torch.arange(b)[:, None, None].expand_as(r)
    hi_ = torch.arange(hq)[None, :, None].expand_as(r)
    got_o = parts[1][0].cpu()[bi, hi_, r].double().numpy()
    got_l = parts[1][1].cpu()[bi, hi_, r].double().numpy()
    assert np.max(np.abs(got_o - o_r)) < 2e-3  # FP32 partial: no BF16 rounding of O
    assert np.max(np.abs(got_l - l_r)) < 1e-3


def test_split_on_side_stream_keeps_its_workspace():
    # The binding allocates the partials workspace itself and drops it on
    # return while the kernels run on a side stream; a same-sized buffer
    # allocated and filled on the default stream right after must not share
    # its memory (else the fill corrupts the partials).
    b, hq, sq, sk, n = 1, 16, 256, 32768, 8
    q, k, v = make_qkv(b, hq, hq, sq, sk, seed=7600)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    want, want_lse = run_split(q, k, v, False, n)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    for _ in range(5):
        o, lse = attn.attn_fwd_split(qd, kd, vd, scale=SCALE, n_splits=n, stream=side)
        junk = torch.empty(attn.split_workspace_bytes(b, hq, sq, n), dtype=torch.uint8,
                           device="cuda")
        junk.fill_(0xFF)  # NaN patterns if it aliased the partials
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        assert torch.equal(o, want) and torch.equal(lse, want_lse)
    assert attn.attn_status() == attn.ATTN_OK


def test_binding_checks_output_tensors():
    q, k, v = make_qkv(1, 2, 2, 256, 256, seed=7700)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    with pytest.raises(ValueError):
        attn.attn_fwd(qd, kd, vd, o=torch.empty(1, 128, 2, 128, dtype=torch.bfloat16,
                                                device="cuda"))
    with pytest.raises(TypeError):
        attn.attn_fwd(qd, kd, vd, lse=torch.empty(1, 2, 256, dtype=torch.float16, device="cuda"))
    with pytest.raises(ValueError):
        attn.attn_fwd_partials(qd, kd, vd, o_part=torch.empty(1, 2, 255, 128, device="cuda"))
    with pytest.raises(ValueError):
        attn.attn_fwd_split(qd, kd, vd, n_splits=2,
                            lse=torch.empty(1, 256, 2, dtype=torch.float32,
                                            device="cuda").transpose(1, 2))

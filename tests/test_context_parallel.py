"""Context-parallel forward (keys split across ranks): host logic on two CPU
gloo ranks, and the device steps (shard partials with their own causal
diagonal, then the merge) on one GPU against the FP64 oracle.

The reference for every split is the oracle of the whole problem: softmax
over the union of the shards' keys is plain attention over all keys.  A
shard's own partial is the oracle's P restricted to the shard's keys and
renormalised: O_r = sum_{j in shard} P_j V_j / sum_{j in shard} P_j and
LSE_r = LSE + log sum_{j in shard} P_j (-inf when the row sees none of them).
"""
from __future__ import annotations

import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from scaled_dot_product_10_b200.workloads import make_qkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SCALE = 1.0 / math.sqrt(128)


def shard_partial_ref(q, k, v, causal, k0, n):
    """FP64 partial of keys [k0, k0 + n) from the oracle's P of the whole problem."""
    o_full, lse_full, p = oracle.attn_fwd(q, k, v, causal, SCALE, want_p=True)
    w = p[..., k0:k0 + n]                                  # [b, h, s_q, n]
    mass = w.sum(-1)
    group = q.shape[2] // k.shape[2]
    vv = v.double().numpy()[:, k0:k0 + n]                  # [b, n, h_kv, d]
    vv = np.repeat(vv.transpose(0, 2, 1, 3), group, axis=1)  # [b, h_q, n, d]
    with np.errstate(divide="ignore", invalid="ignore"):
        o = np.einsum("bhij,bhjd->bhid", w, vv) / mass[..., None]
        lse = lse_full + np.log(mass)
    o[mass == 0] = 0.0
    lse[mass == 0] = -np.inf
    return o, lse


def merge_ref(o_parts, lse_parts):
    """LSE = log sum_r exp LSE_r, O = sum_r exp(LSE_r - LSE) O_r (FP64)."""
    m = np.max(lse_parts, axis=0)
    wts = np.exp(lse_parts - m)
    lse = m + np.log(wts.sum(0))
    o = (np.exp(lse_parts - lse)[..., None] * o_parts).sum(0)
    return o, lse


# ---------------------------------------------------------------- CPU ranks
def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, lengths, causal, give_offsets, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from scaled_dot_product_10_b200.context_parallel import PartialOps, context_parallel_attn_fwd

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        s_k = sum(lengths)
        q, k, v = make_qkv(1, 4, 2, 96, s_k, seed=8100)
        k0 = sum(lengths[:rank])
        k_sh, v_sh = k[:, k0:k0 + lengths[rank]], v[:, k0:k0 + lengths[rank]]
        seen = {}

        def partials(qq, kk, vv, c, scale, diag):
            seen["diag"] = diag
            assert kk.shape[1] == lengths[rank] and scale == SCALE
            if not c:
                o, lse, _ = oracle.attn_fwd(qq, kk, vv, False, scale)
                return torch.from_numpy(o), torch.from_numpy(lse)
            o, lse = shard_partial_ref(q, k, v, True, k0, lengths[rank])
            return torch.from_numpy(o), torch.from_numpy(lse)

        def merge(o_parts, lse_parts):
            seen["parts"] = lse_parts.numpy().copy()
            o, lse = merge_ref(o_parts.numpy(), lse_parts.numpy())
            return torch.from_numpy(o), torch.from_numpy(lse)

        kw = dict(key_offset=k0, s_k_total=s_k) if give_offsets else {}
        o, lse = context_parallel_attn_fwd(q, k_sh, v_sh, causal=causal, scale=SCALE,
                                           ops=PartialOps(partials, merge), **kw)
        o_ref, lse_ref, _ = oracle.attn_fwd(q, k, v, causal, SCALE)
        out.put((rank, seen["diag"], float(np.max(np.abs(o.numpy() - o_ref))),
                 float(np.max(np.abs(lse.numpy() - lse_ref))), seen["parts"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("causal,give_offsets,lengths", [
    (False, False, [170, 130]), (True, False, [250, 50]), (True, True, [250, 50])])
def test_two_gloo_ranks_gather_in_rank_order_and_merge_to_the_whole(causal, give_offsets,
                                                                    lengths):
    # Uneven shards; under the causal mask query row i sees keys <= i + 204,
    # so rows 0..45 of the 96 queries see no key of the second shard (250..299).
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, lengths, causal, give_offsets, out))
             for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted((out.get(timeout=10) for _ in range(2)), key=lambda t: t[0])
    s_k, s_q = sum(lengths), 96
    for rank, diag, err_o, err_lse, parts in res:
        assert diag == s_k - s_q - sum(lengths[:rank])
        assert err_o < 1e-12 and err_lse < 1e-12
        # parts[r] is rank r's LSE_r on every rank: rank order kept.
        assert np.array_equal(parts, res[0][4], equal_nan=True)
    if causal:
        lse1 = res[0][4][1]
        assert np.all(np.isneginf(lse1[..., :46])) and np.all(np.isfinite(lse1[..., 46:]))
        assert np.all(np.isfinite(res[0][4][0]))


def test_shard_partials_merge_to_the_whole_in_fp64():
    # Pins the test's own references: shard partials from P, merged, give
    # the oracle's whole result (three shards, causal, a shard past every
    # early row's diagonal).
    q, k, v = make_qkv(1, 2, 1, 40, 100, seed=8200)
    parts = [shard_partial_ref(q, k, v, True, k0, n) for k0, n in ((0, 30), (30, 50), (80, 20))]
    o, lse = merge_ref(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    o_ref, lse_ref, _ = oracle.attn_fwd(q, k, v, True, SCALE)
    assert np.max(np.abs(o - o_ref)) < 1e-12 and np.max(np.abs(lse - lse_ref)) < 1e-12
    assert np.isneginf(parts[2][1][0, 0, 0])  # row 0 sees keys <= 60: none of 80..99


# ---------------------------------------------------------------- one GPU
SHARD_SHAPES = [
    (1, 4, 2, 300, (1000, 700, 1300)),      # uneven shards, ragged blocks
    (2, 8, 8, 256, (128, 128, 128, 128)),   # one key block per shard
    (1, 16, 1, 64, (4096, 4096)),           # MQA, few queries, long shards
    (1, 2, 2, 700, (300, 200)),             # s_q > a shard's key count (non-causal only)
]


@pytest.mark.gpu
@pytest.mark.parametrize("b,hq,hkv,s_q,lengths,causal", [
    (*shape, causal) for shape in SHARD_SHAPES for causal in (False, True)
    if not (causal and shape[3] > sum(shape[4]))])  # causal needs s_q <= S_k
def test_gpu_shard_partials_and_merge(b, hq, hkv, s_q, lengths, causal):
    from parity import assert_within, gather_rows, metrics
    from scaled_dot_product_10_b200 import attn

    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    s_k = sum(lengths)
    q, k, v = make_qkv(b, hq, hkv, s_q, s_k, seed=8300 + s_q + s_k)
    qd = q.cuda()
    o_parts, l_parts = [], []
    k0 = 0
    for n in lengths:
        kd, vd = k[:, k0:k0 + n].contiguous().cuda(), v[:, k0:k0 + n].contiguous().cuda()
        o_r, l_r = attn.attn_fwd_partials_shard(qd, kd, vd, causal=causal, scale=SCALE,
                                                diag_offset=attn.shard_diag_offset(s_k, s_q, k0))
        assert attn.attn_status() == attn.ATTN_OK
        want_o, want_l = shard_partial_ref(q, k, v, causal, k0, n)
        got_o, got_l = o_r.cpu().double().numpy(), l_r.cpu().double().numpy()
        empty = np.isneginf(want_l)
        assert np.array_equal(np.isneginf(got_l), empty), "rows with no key of the shard"
        assert np.all(got_o[empty] == 0.0)
        if (~empty).any():
            assert np.max(np.abs(got_l[~empty] - want_l[~empty])) <= 1e-3
            d = got_o[~empty] - want_o[~empty]
            assert np.max(np.abs(d)) <= 2e-2
            assert np.linalg.norm(d) <= 5e-3 * np.linalg.norm(want_o[~empty])
        o_parts.append(o_r)
        l_parts.append(l_r)
        k0 += n
    o, lse = attn.merge_partials(torch.stack(o_parts), torch.stack(l_parts))
    assert attn.attn_status() == attn.ATTN_OK
    o_ref, l_ref, _ = oracle.attn_fwd(q, k, v, causal, SCALE)
    oo, ll = gather_rows(o, lse, None)
    assert_within(metrics(oo, ll, o_ref, l_ref), f"context-parallel shards {lengths}")


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_gpu_wrapper_on_a_one_rank_nccl_group(causal):
    # The wrapper end to end with the CUDA steps and the NCCL all-gather, on
    # a process group of one rank (this pool gives one GPU per call).
    import torch.distributed as dist

    from parity import assert_within, gather_rows, metrics
    from scaled_dot_product_10_b200.context_parallel import context_parallel_attn_fwd

    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, store=dist.HashStore(),
                            device_id=torch.device("cuda", 0))
    try:
        q, k, v = make_qkv(2, 8, 2, 500, 1500, seed=8400)
        o, lse = context_parallel_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal,
                                           scale=SCALE)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    o_ref, l_ref, _ = oracle.attn_fwd(q, k, v, causal, SCALE)
    oo, ll = gather_rows(o, lse, None)
    assert_within(metrics(oo, ll, o_ref, l_ref), "context-parallel wrapper, one rank")

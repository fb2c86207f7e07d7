"""GPU parity: the CUDA path against the FP64 oracle on identical seeded
BF16 inputs (B200 only)."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from parity import assert_within, check, gather_rows, metrics, run_gpu
from scaled_dot_product_10_b200 import attn
from scaled_dot_product_10_b200.workloads import WORKLOADS, make_qkv, sample_rows, workload_qkv

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    attn.load_library()


# ----------------------------------------------------------------- small cases
@pytest.mark.parametrize("causal", [False, True])
def test_tiny_config(causal):
    w = WORKLOADS["tiny_b1_h2_s256"]
    q, k, v = workload_qkv(w)
    check(q, k, v, causal, w.scale, what=f"{w.name} causal={causal}")


# Sequence tails (not multiples of the 128-row tile), single rows, one head.
@pytest.mark.parametrize("s", [1, 2, 64, 127, 128, 129, 200, 255, 383, 640, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_tails(s, causal):
    q, k, v = make_qkv(1, 1, 1, s, s, seed=2000 + s)
    check(q, k, v, causal, SCALE, what=f"s={s} causal={causal}")


@pytest.mark.parametrize("s_q,s_k", [(1, 300), (300, 1), (128, 1024), (777, 129), (64, 4096)])
def test_noncausal_rectangular(s_q, s_k):
    q, k, v = make_qkv(2, 4, 2, s_q, s_k, seed=3000 + s_q + s_k)
    check(q, k, v, False, SCALE, what=f"s_q={s_q} s_k={s_k}")


@pytest.mark.parametrize("b,hq,hkv,s_q,s_k", [
    (1, 4, 4, 100, 1000),    # bottom-right diagonal inside a key block
    (1, 2, 2, 129, 1000),    # ragged queries, two query blocks
    (2, 8, 2, 384, 4096),    # GQA, three query blocks (an odd pair)
    (1, 16, 16, 1, 4096),    # one query row (decode) sees every key
    (1, 4, 1, 640, 643),     # offset 3: diagonal blocks straddle key blocks
])
def test_causal_rectangular(b, hq, hkv, s_q, s_k):
    # Causal with fewer queries than keys: query i sees keys 0 .. i + s_k - s_q.
    q, k, v = make_qkv(b, hq, hkv, s_q, s_k, seed=6800 + s_q + s_k)
    rows = None if b * hq * s_q <= 8192 else sample_rows(b, hq, s_q, 64, seed=6801)
    check(q, k, v, True, SCALE, rows=rows, what=f"causal {s_q}x{s_k}")


@pytest.mark.parametrize("h_q,h_kv", [(16, 2), (16, 1), (8, 8), (6, 3), (4, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_head_sharing_small(h_q, h_kv, causal):
    q, k, v = make_qkv(2, h_q, h_kv, 384, 384, seed=4000 + h_q * 10 + h_kv)
    check(q, k, v, causal, SCALE, what=f"h_q={h_q} h_kv={h_kv} causal={causal}")


@pytest.mark.parametrize("scale", [1e-3, 0.05, 0.5, 2.0])
def test_scales(scale):
    q, k, v = make_qkv(1, 2, 2, 512, 512, seed=5000)
    check(q, k, v, True, scale, what=f"scale={scale}")


@pytest.mark.parametrize("scale", [-0.09, -1.0, 0.0, -0.0])
@pytest.mark.parametrize("causal", [False, True])
def test_negative_and_zero_scale(scale, causal):
    # The formula puts no condition on the scale.  A negative scale favours
    # the keys least aligned with the query; scale 0 gives uniform weights
    # over the visible keys (LSE = ln of their count).
    q, k, v = make_qkv(2, 4, 2, 300, 700, seed=5100)
    check(q, k, v, causal, scale, what=f"scale={scale} causal={causal}")


def test_rescale_branch_forced():
    # Keys whose scores beat every earlier key block's maximum by much more
    # than 2^8 in the exponent force the running output to be rescaled
    # (twice per row: at key 300 and again at key 450); key 200 raises the
    # maximum by less than 2^8, which must not rescale.  Every row's result
    # then depends on the correction being applied exactly: a skipped or
    # doubled correction weighs the early keys wrong by a factor > 2^16.
    b, h, s = 1, 2, 512
    g = torch.Generator().manual_seed(6250)
    q = (1.0 + 0.1 * torch.randn(b, s, h, 128, generator=g)).to(torch.bfloat16)
    k = 0.1 * torch.randn(b, s, h, 128, generator=g)
    k[:, 200] = 0.4   # score ~ 51 * scale -> exponent ~ 6.5 above block 0
    k[:, 300] = 1.0   # ~ 128 * scale -> ~ 16 above
    k[:, 450] = 2.0   # ~ 256 * scale -> another ~ 16
    k = k.to(torch.bfloat16)
    v = torch.randn(b, s, h, 128, generator=g).to(torch.bfloat16)
    for causal in (False, True):
        check(q, k, v, causal, SCALE, what=f"forced rescale causal={causal}")


def test_many_tiles_more_than_sms():
    # 2 * 8 * 12 = 192 tiles > 148 SMs: exercises the persistent loop and the
    # reuse of TMEM, barriers and the Q double buffer across tiles.
    q, k, v = make_qkv(2, 8, 4, 1536, 1536, seed=6000)
    for causal in (False, True):
        check(q, k, v, causal, SCALE, what=f"persistent causal={causal}")


def test_uniform_distribution_inputs():
    q, k, v = make_qkv(2, 4, 4, 700, 700, seed=6100, dist="uniform")
    for causal in (False, True):
        check(q, k, v, causal, SCALE, what=f"uniform causal={causal}")


def test_large_logits_sharp_softmax():
    # K x 8: scores up to ~90 in magnitude; exercises the rescale path.
    q, k, v = make_qkv(1, 2, 2, 1024, 1024, seed=6200, k_scale=8.0)
    for causal in (False, True):
        check(q, k, v, causal, SCALE, what=f"sharp causal={causal}")


def test_identical_v_rows_exact():
    # The weights of a row sum to one, so identical V rows come back up to
    # BF16 rounding of O itself.
    q, k, _ = make_qkv(1, 2, 2, 384, 384, seed=6300)
    vrow = torch.randn(1, 1, 2, 128).to(torch.bfloat16)
    v = vrow.expand(1, 384, 2, 128).contiguous()
    o, _ = run_gpu(q, k, v, False, SCALE)
    want = vrow.float().expand(1, 384, 2, 128)
    assert torch.max(torch.abs(o.float().cpu() - want)) <= 2 * 2 ** -8 * want.abs().max()


def test_deterministic():
    q, k, v = make_qkv(2, 4, 2, 1000, 1000, seed=6400)
    o1, l1 = run_gpu(q, k, v, True, SCALE)
    o2, l2 = run_gpu(q, k, v, True, SCALE)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("s", [4096, 3968, 1152])
def test_causal_turn_order_many_launches(s):
    # In a causal pair the second query block has one key block more than
    # the first, and an odd block count leaves the last pair's second block
    # empty.  The two softmax warpgroups' turn order on the exponential unit
    # must survive both over many launches: a lost turn ends in the bounded
    # wait's timeout status, and every launch must give the same bits.
    b, h = 2, 16
    q, k, v = make_qkv(b, h, h, s, s, seed=6450 + s)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o0, l0 = run_gpu(q, k, v, True, SCALE)
    o, lse = torch.empty_like(o0), torch.empty_like(l0)
    for i in range(200):
        attn.attn_fwd(qd, kd, vd, causal=True, scale=SCALE, o=o, lse=lse)
        if i % 50 == 49:
            assert attn.attn_status() == attn.ATTN_OK, f"launch {i}"
            assert torch.equal(o, o0) and torch.equal(lse, l0), f"launch {i}"
    rows = sample_rows(b, h, s, 64, seed=6460 + s)
    o_ref, l_ref, _ = oracle.attn_fwd(q, k, v, True, SCALE, rows=rows)
    oo, ll = gather_rows(o0, l0, rows)
    assert_within(metrics(oo, ll, o_ref, l_ref), f"causal s={s}")


def test_outputs_stay_in_bounds():
    # o and lse sit inside larger buffers; the guard regions must be untouched.
    b, h, s = 1, 2, 200
    q, k, v = make_qkv(b, h, h, s, s, seed=6500)
    pad = 4096
    o_buf = torch.full((pad * 2 + b * s * h * 128,), 1234.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((pad * 2 + b * h * s,), -7.0, dtype=torch.float32, device="cuda")
    o = o_buf[pad:pad + b * s * h * 128].view(b, s, h, 128)
    lse = l_buf[pad:pad + b * h * s].view(b, h, s)
    attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, scale=SCALE, o=o, lse=lse)
    assert attn.attn_status() == attn.ATTN_OK
    assert torch.all(o_buf[:pad] == 1234.0) and torch.all(o_buf[-pad:] == 1234.0)
    assert torch.all(l_buf[:pad] == -7.0) and torch.all(l_buf[-pad:] == -7.0)
    o_ref, l_ref, _ = oracle.attn_fwd(q, k, v, True, SCALE)
    oo, ll = gather_rows(o, lse, None)
    assert_within(metrics(oo, ll, o_ref, l_ref), "guarded")


def test_host_buffer_entry_point():
    b, hq, hkv, s = 2, 4, 2, 513
    q, k, v = make_qkv(b, hq, hkv, s, s, seed=6600)
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((b, hq, s), dtype=torch.float32).pin_memory()
    ws = torch.empty(attn.host_workspace_bytes(b, hq, hkv, s, s), dtype=torch.uint8, device="cuda")
    attn.attn_fwd_host(qh, kh, vh, oh, lh, ws, causal=True, scale=SCALE)
    assert attn.attn_status() == attn.ATTN_OK
    o_ref, l_ref, _ = oracle.attn_fwd(q, k, v, True, SCALE)
    oo, ll = gather_rows(oh, lh, None)
    assert_within(metrics(oo, ll, o_ref, l_ref), "host entry")


@pytest.mark.parametrize("b,hq,hkv,s", [
    (1, 16, 16, 8192),  # four groups of 4 key/value heads
    (2, 12, 6, 4096),   # three groups of 2 (GQA)
    (1, 10, 5, 8192),   # two uneven groups (3 and 2 key/value heads)
])
def test_host_buffer_pipelined_groups(b, hq, hkv, s):
    """Large problems go through the host entry in groups of key/value heads
    whose copies overlap the kernel of another group: every output must be
    bit-identical to the device entry on the same inputs.  Two calls are
    queued back to back on one workspace with different inputs, so the
    second call's copies in must wait for the first call's kernels."""
    q, k, v = make_qkv(b, hq, hkv, s, s, seed=6650 + hq)
    q2 = make_qkv(b, hq, hkv, s, s, seed=6660 + hq)[0]
    qh, q2h, kh, vh = q.pin_memory(), q2.pin_memory(), k.pin_memory(), v.pin_memory()
    outs = [(torch.empty_like(qh).pin_memory(),
             torch.empty((b, hq, s), dtype=torch.float32).pin_memory()) for _ in range(2)]
    ws = torch.empty(attn.host_workspace_bytes(b, hq, hkv, s, s), dtype=torch.uint8, device="cuda")
    attn.attn_fwd_host(qh, kh, vh, outs[0][0], outs[0][1], ws, causal=False, scale=SCALE)
    attn.attn_fwd_host(q2h, kh, vh, outs[1][0], outs[1][1], ws, causal=True, scale=SCALE)
    assert attn.attn_status() == attn.ATTN_OK
    kd, vd = k.cuda(), v.cuda()
    for (oh, lh), qq, causal in ((outs[0], q, False), (outs[1], q2, True)):
        o_dev, l_dev = attn.attn_fwd(qq.cuda(), kd, vd, causal=causal, scale=SCALE)
        assert attn.attn_status() == attn.ATTN_OK
        assert torch.equal(oh, o_dev.cpu()), f"O differs (causal={causal})"
        assert torch.equal(lh, l_dev.cpu()), f"LSE differs (causal={causal})"
    rows = sample_rows(b, hq, s, 64, seed=6670 + hq)
    o_ref, l_ref, _ = oracle.attn_fwd(q2, k, v, True, SCALE, rows=rows)
    oo, ll = gather_rows(outs[1][0], outs[1][1], rows)
    assert_within(metrics(oo, ll, o_ref, l_ref), "host entry, groups")


def test_bounded_wait_reports_timeout_and_context_survives():
    assert attn.attn_status() == attn.ATTN_OK
    assert attn.selftest_wait_timeout(50_000_000) == attn.ATTN_OK  # 50 ms
    assert attn.attn_status() == attn.ATTN_ERR_TIMEOUT
    assert attn.attn_status() == attn.ATTN_OK  # the word was cleared
    q, k, v = make_qkv(1, 2, 2, 256, 256, seed=6700)
    check(q, k, v, False, SCALE, what="after timeout self-test")


# ------------------------------------------------------- the workload configs
def _rows_for(w, n):
    return sample_rows(w.batch, w.h_q, w.seq, n, seed=w.seed + 7919)


FULL = ["tiny_b1_h2_s256", "mha_b8_h16_s4096", "gqa_b8_h16_kv2_s2048", "mqa_b8_h16_kv1_s2048"]
SAMPLED = ["mha_b4_h16_s8192", "mha_b2_h16_s16384", "mha_b1_h16_s32768_k3"]


@pytest.mark.parametrize("name", FULL + SAMPLED)
@pytest.mark.parametrize("causal", [False, True])
def test_workload_configs(name, causal):
    """Every config at full size, in the launch configuration the bench
    times.  The oracle evaluates every query row of the 256-, 2K- and
    4K-sequence configs, and 512 sampled query rows per head of the 8K-32K
    ones (always including rows 0, 1, 127, 128, 255, 256 and s-1)."""
    w = WORKLOADS[name]
    q, k, v = workload_qkv(w)
    rows = _rows_for(w, 512) if w.sampled else None
    m = check(q, k, v, causal, w.scale, rows=rows, what=f"{name} causal={causal}")
    print(name, causal, m)


# ------------------------------------------------------------ sliding window
def check_window(q, k, v, w, scale=SCALE, rows=None, what=""):
    o, lse = attn.attn_fwd_window(q.cuda(), k.cuda(), v.cuda(), w, scale=scale)
    rc = attn.attn_status()
    assert rc == attn.ATTN_OK, attn.attn_strerror(rc)
    o_ref, l_ref, _ = oracle.attn_fwd(q, k, v, True, scale, rows=rows, window_left=w)
    oo, ll = gather_rows(o, lse, rows)
    m = metrics(oo, ll, o_ref, l_ref)
    assert_within(m, what)
    return o, lse


@pytest.mark.parametrize("s_q,s_k,w", [
    (1000, 1000, 0), (1000, 1000, 1), (1000, 1000, 127), (1000, 1000, 128),
    (1000, 1000, 129), (1000, 1000, 300), (640, 640, 255), (129, 129, 64),
    (300, 1000, 100),   # bottom-right: the window slides with the offset
    (1, 4096, 500),     # one query row
    (2048, 2048, 2047), # the window covers every visible key
])
def test_window_matches_oracle(s_q, s_k, w):
    q, k, v = make_qkv(2, 4, 2, s_q, s_k, seed=9000 + s_q + w)
    check_window(q, k, v, w, what=f"window {s_q}x{s_k} w={w}")


@pytest.mark.parametrize("h_q,h_kv", [(16, 2), (16, 1)])
def test_window_head_sharing(h_q, h_kv):
    q, k, v = make_qkv(2, h_q, h_kv, 2048, 2048, seed=9100 + h_kv)
    rows = sample_rows(2, h_q, 2048, 128, seed=9101)
    check_window(q, k, v, 511, rows=rows, what=f"window gqa {h_q}/{h_kv}")


def test_window_wider_than_keys_is_causal_bit_exact():
    q, k, v = make_qkv(1, 4, 4, 700, 700, seed=9200)
    o1, l1 = run_gpu(q, k, v, True, SCALE)
    o2, l2 = attn.attn_fwd_window(q.cuda(), k.cuda(), v.cuda(), 5000, scale=SCALE)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("s,w", [(4096, 1000), (3968, 300), (1152, 129)])
def test_window_turn_order_many_launches(s, w):
    # Windowed pairs take turns only over the key blocks both query blocks
    # visit; 100 launches must give a clean status word and identical bits.
    b, h = 2, 16
    q, k, v = make_qkv(b, h, h, s, s, seed=9300 + s)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o0, l0 = attn.attn_fwd_window(qd, kd, vd, w, scale=SCALE)
    o, lse = torch.empty_like(o0), torch.empty_like(l0)
    for i in range(100):
        attn.attn_fwd_window(qd, kd, vd, w, scale=SCALE, o=o, lse=lse)
        if i % 50 == 49:
            assert attn.attn_status() == attn.ATTN_OK, f"launch {i}"
            assert torch.equal(o, o0) and torch.equal(lse, l0), f"launch {i}"
    rows = sample_rows(b, h, s, 64, seed=9310 + s)
    o_ref, l_ref, _ = oracle.attn_fwd(q, k, v, True, SCALE, rows=rows, window_left=w)
    oo, ll = gather_rows(o0, l0, rows)
    assert_within(metrics(oo, ll, o_ref, l_ref), f"window s={s} w={w}")

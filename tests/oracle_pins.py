"""Pins that tie the FP64 oracle to facts fixed by the definition.

Every pin takes the loaded oracle library (the real one, or a planted
mutant in the mutation test) and raises AssertionError when the oracle
disagrees with what the definition ``softmax(Q K^T * scale) V`` fixes
(rkmt.cn page, section 1; the three steps of the bjdmk.com.cn page,
section 1; the causal mask of the intelliparadigm.com AVO page,
section 2.2; grouped heads, rkmt.cn page section 3.2).

None of these re-types the oracle's formula: each compares against a
closed form, an invariant of the definition, a hand derivation, or an
independent library routine (torch's float64 SDPA on the CPU).
"""
from __future__ import annotations

import glob
import json
import math
import os

import numpy as np
import scipy.special
import torch

import oracle
from scaled_dot_product_10_b200.workloads import make_qkv

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def bf16(a) -> torch.Tensor:
    """Exact BF16 tensor from values that BF16 represents exactly."""
    t = torch.as_tensor(np.asarray(a, dtype=np.float64)).to(torch.bfloat16)
    back = t.to(torch.float64).numpy()
    assert np.array_equal(back, np.asarray(a, dtype=np.float64)), "value not exact in bf16"
    return t


def f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def grid_values(rng, shape, lo=-2.0, hi=2.0, step=0.125):
    """Random multiples of ``step`` in [lo, hi]: exact in BF16, and sums or
    integer multiples of them stay exact."""
    n = int(round((hi - lo) / step))
    return lo + step * rng.integers(0, n + 1, size=shape)


def run(lib, q, k, v, causal, scale, rows=None, want_p=False):
    return oracle.attn_fwd(q, k, v, causal, scale, rows=rows, want_p=want_p, lib=lib)


def run_w(lib, q, k, v, scale, window_left):
    """Causal with a sliding window of window_left keys before the diagonal."""
    return oracle.attn_fwd(q, k, v, True, scale, lib=lib, window_left=window_left)


# ---------------------------------------------------------------------------


def pin_rows_sum_to_one(lib):
    """Softmax normalisation: each row of P sums to 1; masked entries are 0."""
    q, k, v = make_qkv(1, 2, 2, 37, 37, seed=11, d=16)
    for causal in (False, True):
        _, _, p = run(lib, q, k, v, causal, 0.25, want_p=True)
        assert np.all(np.abs(p.sum(-1) - 1.0) < 1e-12), "rows of P do not sum to 1"
        assert np.all(p >= 0.0)
        if causal:
            i = np.arange(37)[:, None]
            j = np.arange(37)[None, :]
            assert np.all(p[..., j > i] == 0.0), "causal P is non-zero above the diagonal"
            assert np.all(p[..., j <= i] > 0.0)


def pin_identical_v_rows(lib):
    """If every V row of a head equals v, the output of every query is v."""
    rng = np.random.default_rng(5)
    b, s, h_q, h_kv, d = 2, 19, 4, 2, 8
    q, k, _ = make_qkv(b, h_q, h_kv, s, s, seed=12, d=d)
    vrow = grid_values(rng, (b, 1, h_kv, d))
    v = bf16(np.broadcast_to(vrow, (b, s, h_kv, d)).copy())
    for causal in (False, True):
        o, _, _ = run(lib, q, k, v, causal, 1 / math.sqrt(d))
        for h in range(h_q):
            g = h // (h_q // h_kv)
            want = vrow[:, 0, g, :][:, None, :]
            assert np.max(np.abs(o[:, h] - want)) < 1e-12, "identical V rows not reproduced"


def pin_zero_query(lib):
    """Q = 0 makes every visible score 0: O is the mean of the visible V rows
    and LSE = ln(#visible keys) (s_k non-causal, i+1 causal)."""
    b, s, h, d = 1, 29, 2, 8
    _, k, v = make_qkv(b, h, h, s, s, seed=13, d=d)
    q = torch.zeros((b, s, h, d), dtype=torch.bfloat16)
    vv = f64(v)
    o, lse, _ = run(lib, q, k, v, False, 0.3)
    want = vv.mean(axis=1)  # [b, h, d]
    assert np.max(np.abs(o - want[:, :, None, :])) < 1e-12, "Q=0: O is not the mean of V"
    assert np.max(np.abs(lse - math.log(s))) < 1e-12, "Q=0: LSE is not ln(s_k)"
    o, lse, _ = run(lib, q, k, v, True, 0.3)
    for i in range(s):
        want_i = vv[:, : i + 1].mean(axis=1)
        assert np.max(np.abs(o[:, :, i] - want_i)) < 1e-12, "Q=0 causal: O is not the prefix mean"
        assert np.max(np.abs(lse[:, :, i] - math.log(i + 1))) < 1e-12, "Q=0 causal: LSE != ln(i+1)"


def pin_causal_row0(lib):
    """Causal row 0 sees only key 0: O_0 = V_0 and LSE_0 = scale * q_0 . k_0."""
    b, s, h, d = 2, 23, 3, 16
    q, k, v = make_qkv(b, h, h, s, s, seed=14, d=d)
    scale = 0.177
    o, lse, _ = run(lib, q, k, v, True, scale)
    qq, kk, vv = f64(q), f64(k), f64(v)
    for bi in range(b):
        for hi in range(h):
            assert np.max(np.abs(o[bi, hi, 0] - vv[bi, 0, hi])) < 1e-12, "causal row 0 != V_0"
            want = scale * float(np.dot(qq[bi, 0, hi], kk[bi, 0, hi]))
            assert abs(lse[bi, hi, 0] - want) < 1e-12, "causal LSE_0 != scale q0.k0"


def pin_causal_rectangular_is_square_suffix(lib):
    """Causal with s_q < s_k (bottom-right alignment): the s_q queries are the
    last s_q rows of a square causal problem over the same keys, so their O
    and LSE equal those rows of the square result (pinned above)."""
    b, h, s_k, s_q, d = 1, 2, 19, 7, 8
    q_full, k, v = make_qkv(b, h, h, s_k, s_k, seed=41, d=d)
    q = q_full[:, s_k - s_q:].contiguous()
    o_sq, l_sq, _ = run(lib, q_full, k, v, True, 0.31)
    o, l, _ = run(lib, q, k, v, True, 0.31)
    assert np.max(np.abs(o - o_sq[:, :, s_k - s_q:])) < 1e-12, "rectangular causal != square suffix"
    assert np.max(np.abs(l - l_sq[:, :, s_k - s_q:])) < 1e-12, "rectangular causal LSE != square suffix"


def pin_causal_single_query_sees_every_key(lib):
    """One query row under the bottom-right causal mask sees all s_k keys:
    the result equals the non-causal one."""
    q, k, v = make_qkv(2, 2, 1, 1, 13, seed=42, d=8)
    o_c, l_c, _ = run(lib, q, k, v, True, 0.5)
    o_n, l_n, _ = run(lib, q, k, v, False, 0.5)
    assert np.max(np.abs(o_c - o_n)) < 1e-12 and np.max(np.abs(l_c - l_n)) < 1e-12, \
        "single causal query does not see every key"


def pin_window_covering_every_key_is_causal(lib):
    """A sliding window at least as wide as the key sequence removes nothing
    the causal mask keeps."""
    q, k, v = make_qkv(1, 2, 2, 9, 17, seed=43, d=8)
    o_w, l_w, _ = run_w(lib, q, k, v, 0.37, 17)
    o_c, l_c, _ = run(lib, q, k, v, True, 0.37)
    assert np.max(np.abs(o_w - o_c)) < 1e-12 and np.max(np.abs(l_w - l_c)) < 1e-12, \
        "full-width window differs from causal"


def pin_window_zero_keeps_the_diagonal_key(lib):
    """window_left = 0: row i sees only key i + s_k - s_q, so O_i is that V row
    and LSE_i = scale * q_i . k_(i + s_k - s_q)."""
    b, h, s_q, s_k, d = 1, 2, 6, 10, 8
    q, k, v = make_qkv(b, h, h, s_q, s_k, seed=44, d=d)
    scale = 0.29
    o, lse, _ = run_w(lib, q, k, v, scale, 0)
    qq, kk, vv = f64(q), f64(k), f64(v)
    for hi in range(h):
        for i in range(s_q):
            j = i + s_k - s_q
            assert np.max(np.abs(o[0, hi, i] - vv[0, j, hi])) < 1e-12, "window 0: O != V_diag"
            want = scale * float(np.dot(qq[0, i, hi], kk[0, j, hi]))
            assert abs(lse[0, hi, i] - want) < 1e-12, "window 0: LSE != scale q.k_diag"


def pin_window_row_is_attention_over_its_keys(lib):
    """Row i under a window of W sees exactly the keys lo..hi with
    hi = i + s_k - s_q and lo = max(0, hi - W): its O and LSE equal plain
    (non-causal) attention of that row over K[lo:hi+1], V[lo:hi+1]."""
    b, h, s_q, s_k, d, W = 1, 2, 12, 15, 8, 4
    q, k, v = make_qkv(b, h, 1, s_q, s_k, seed=45, d=d)
    o, lse, _ = run_w(lib, q, k, v, 0.41, W)
    for i in (0, 1, 5, 11):
        hi = i + s_k - s_q
        lo = max(0, hi - W)
        o1, l1, _ = run(lib, q[:, i:i + 1].contiguous(), k[:, lo:hi + 1].contiguous(),
                        v[:, lo:hi + 1].contiguous(), False, 0.41)
        assert np.max(np.abs(o[:, :, i] - o1[:, :, 0])) < 1e-12, "window row != attention over its keys"
        assert np.max(np.abs(lse[:, :, i] - l1[:, :, 0])) < 1e-12, "window LSE != attention over its keys"


def pin_key_split_merge(lib):
    """Softmax over a key set cut into two ranges: with (O_r, LSE_r) the
    results over each range, LSE = log(exp LSE_1 + exp LSE_2) and
    O = sum_r exp(LSE_r - LSE) O_r reproduce the whole set's O and LSE."""
    q, k, v = make_qkv(2, 3, 1, 5, 14, seed=46, d=8)
    o, lse, _ = run(lib, q, k, v, False, 0.33)
    o1, l1, _ = run(lib, q, k[:, :6].contiguous(), v[:, :6].contiguous(), False, 0.33)
    o2, l2, _ = run(lib, q, k[:, 6:].contiguous(), v[:, 6:].contiguous(), False, 0.33)
    m = np.maximum(l1, l2)
    lse_m = m + np.log(np.exp(l1 - m) + np.exp(l2 - m))
    o_m = np.exp(l1 - lse_m)[..., None] * o1 + np.exp(l2 - lse_m)[..., None] * o2
    assert np.max(np.abs(lse_m - lse)) < 1e-12, "key-range LSEs do not combine to the LSE"
    assert np.max(np.abs(o_m - o)) < 1e-12, "key-range outputs do not combine to O"


def pin_key_shift(lib):
    """Adding one vector c to every key row adds scale*q_i.c to every score of
    row i: O is unchanged and LSE_i moves by scale*q_i.c (both modes)."""
    rng = np.random.default_rng(6)
    b, s, h, d = 1, 21, 2, 8
    q = bf16(grid_values(rng, (b, s, h, d)))
    kk = grid_values(rng, (b, s, h, d))
    c = rng.integers(-2, 3, size=(b, 1, h, d)).astype(np.float64)
    k0, k1 = bf16(kk), bf16(kk + c)
    v = bf16(grid_values(rng, (b, s, h, d)))
    scale = 0.25
    qq = f64(q)
    for causal in (False, True):
        o0, l0, _ = run(lib, q, k0, v, causal, scale)
        o1, l1, _ = run(lib, q, k1, v, causal, scale)
        assert np.max(np.abs(o1 - o0)) < 1e-12, "key shift changed O"
        shift = scale * np.einsum("bshd,bhd->bhs", qq, c[:, 0])
        assert np.max(np.abs((l1 - l0) - shift)) < 1e-10, "key shift did not move LSE by scale*q.c"


def pin_value_affine(lib):
    """O is affine in V with weights summing to 1: V -> 2V + 1 gives O -> 2O + 1."""
    rng = np.random.default_rng(7)
    b, s, h, d = 1, 17, 2, 8
    q, k, _ = make_qkv(b, h, h, s, s, seed=15, d=d)
    vv = grid_values(rng, (b, s, h, d))
    for causal in (False, True):
        o0, l0, _ = run(lib, q, k, bf16(vv), causal, 0.4)
        o1, l1, _ = run(lib, q, k, bf16(2 * vv + 1), causal, 0.4)
        assert np.max(np.abs(o1 - (2 * o0 + 1))) < 1e-12, "O is not affine in V"
        assert np.array_equal(l0, l1), "LSE depends on V"


def pin_key_permutation(lib):
    """Non-causal attention is a sum over keys: permuting the (K, V) rows
    jointly changes neither O nor LSE."""
    b, s, h, d = 2, 31, 2, 16
    q, k, v = make_qkv(b, h, h, s, s, seed=16, d=d)
    perm = torch.as_tensor(np.random.default_rng(8).permutation(s))
    o0, l0, _ = run(lib, q, k, v, False, 0.25)
    o1, l1, _ = run(lib, q, k[:, perm].contiguous(), v[:, perm].contiguous(), False, 0.25)
    assert np.max(np.abs(o1 - o0)) < 1e-12 and np.max(np.abs(l1 - l0)) < 1e-12, \
        "key permutation changed the result"


def pin_gqa_equals_repeated_mha(lib):
    """Grouped heads: h_q query heads over h_kv key/value heads equal plain
    multi-head attention with each K/V head repeated h_q/h_kv times in a row."""
    b, s, h_q, d = 2, 33, 8, 16
    for h_kv in (2, 1):
        q, k, v = make_qkv(b, h_q, h_kv, s, s, seed=17 + h_kv, d=d)
        rep = h_q // h_kv
        k_m = k.repeat_interleave(rep, dim=2).contiguous()
        v_m = v.repeat_interleave(rep, dim=2).contiguous()
        for causal in (False, True):
            o0, l0, _ = run(lib, q, k, v, causal, 0.25)
            o1, l1, _ = run(lib, q, k_m, v_m, causal, 0.25)
            assert np.array_equal(o0, o1) and np.array_equal(l0, l1), "GQA != repeated MHA"


def pin_torch_sdpa_f64(lib):
    """Independent library routine: torch's float64 CPU scaled_dot_product_attention
    (with is_causal and enable_gqa) gives the same O; the LSE matches
    scipy's logsumexp of the library matmul's scaled scores.  (torch's own
    CPU logsumexp is not used: on bit-identical float64 scores it returned a
    result 4.6e-10 off in about one process in twenty.)"""
    cases = [(2, 4, 4, 67, 16), (1, 4, 2, 45, 128), (2, 8, 1, 40, 32)]
    for b, h_q, h_kv, s, d in cases:
        q, k, v = make_qkv(b, h_q, h_kv, s, s, seed=100 + s, d=d)
        scale = 1 / math.sqrt(d)
        qt = q.to(torch.float64).transpose(1, 2)
        kt = k.to(torch.float64).transpose(1, 2)
        vt = v.to(torch.float64).transpose(1, 2)
        for causal in (False, True):
            want = torch.nn.functional.scaled_dot_product_attention(
                qt, kt, vt, is_causal=causal, scale=scale, enable_gqa=(h_q != h_kv))
            o, lse, _ = run(lib, q, k, v, causal, scale)
            assert np.max(np.abs(o - want.numpy())) < 1e-10, "O disagrees with torch SDPA (f64)"
            kr = kt.repeat_interleave(h_q // h_kv, dim=1)
            sc = torch.matmul(qt, kr.transpose(-1, -2)) * scale
            if causal:
                sc = sc.masked_fill(torch.ones(s, s, dtype=torch.bool).triu(1), float("-inf"))
            want_lse = scipy.special.logsumexp(sc.numpy(), axis=-1)
            assert np.max(np.abs(lse - want_lse)) < 1e-10, "LSE disagrees with scipy's logsumexp"


def _closed_form(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"e": math.e, "log": math.log, "exp": math.exp}))


def pin_golden_closed_forms(lib):
    """Hand-derived tiny cases stored under tests/golden (each cites its passage)."""
    files = sorted(glob.glob(os.path.join(GOLDEN, "*.json")))
    assert files, "no golden fixtures"
    for path in files:
        with open(path) as f:
            g = json.load(f)
        q, k, v = bf16(g["q"]), bf16(g["k"]), bf16(g["v"])
        o, lse, _ = oracle.attn_fwd(q, k, v, g["causal"], g["scale"], lib=lib,
                                    window_left=g.get("window_left", -1))
        want_o = np.vectorize(_closed_form)(np.array(g["expected_o"], dtype=object)).astype(np.float64)
        want_l = np.vectorize(_closed_form)(np.array(g["expected_lse"], dtype=object)).astype(np.float64)
        assert np.max(np.abs(o - want_o)) < 1e-14, f"{os.path.basename(path)}: O"
        assert np.max(np.abs(lse - want_l)) < 1e-14, f"{os.path.basename(path)}: LSE"


def pin_row_subset(lib):
    """Evaluating a subset of rows gives those rows of the full evaluation."""
    b, s, h, d = 1, 50, 2, 16
    q, k, v = make_qkv(b, h, h, s, s, seed=21, d=d)
    rows = np.array([[[0, 7, 31, 49], [3, 4, 5, 48]]], dtype=np.int32)
    for causal in (False, True):
        of, lf, _ = run(lib, q, k, v, causal, 0.2)
        os_, ls, _ = run(lib, q, k, v, causal, 0.2, rows=rows)
        for hi in range(h):
            assert np.array_equal(os_[0, hi], of[0, hi, rows[0, hi]])
            assert np.array_equal(ls[0, hi], lf[0, hi, rows[0, hi]])




def _varlen_case(seed, lens_q, lens_k, h_q=4, h_kv=2, d=16):
    """Packed q [total_q, h_q, d], k/v [total_k, h_kv, d] and cu_seqlens."""
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    q, k, v = make_qkv(1, h_q, h_kv, int(cu_q[-1]), int(cu_k[-1]), seed=seed, d=d)
    return q[0], k[0], v[0], cu_q, cu_k


def pin_varlen_matches_block_diagonal_sdpa(lib):
    """A packed batch equals ONE attention over all packed tokens whose mask
    forbids every (query, key) pair of different sequences (and, causal,
    keys past the row's own diagonal in its sequence; with a window of W,
    also keys more than W before that diagonal): torch's float64 SDPA with
    that explicit boolean mask, and scipy's logsumexp of the masked scores."""
    lens_q, lens_k = [5, 1, 9, 3], [7, 4, 9, 3]
    q, k, v, cu_q, cu_k = _varlen_case(31, lens_q, lens_k)
    h_q, h_kv = q.shape[1], k.shape[1]
    seq_q = np.repeat(np.arange(4), lens_q)
    seq_k = np.repeat(np.arange(4), lens_k)
    pos_q = np.arange(cu_q[-1]) - cu_q[seq_q]
    pos_k = np.arange(cu_k[-1]) - cu_k[seq_k]
    off = (np.asarray(lens_k) - np.asarray(lens_q))[seq_q]
    for causal, window in ((False, -1), (True, -1), (True, 0), (True, 3)):
        allow = seq_q[:, None] == seq_k[None, :]
        if causal:
            allow &= pos_k[None, :] <= (pos_q + off)[:, None]
        if window >= 0:
            allow &= pos_k[None, :] >= (pos_q + off - window)[:, None]
        mask = torch.from_numpy(allow)
        qt = q.double().permute(1, 0, 2)[None]                    # [1, h_q, Tq, d]
        kt = k.double().permute(1, 0, 2).repeat_interleave(h_q // h_kv, 0)[None]
        vt = v.double().permute(1, 0, 2).repeat_interleave(h_q // h_kv, 0)[None]
        want = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask,
                                                                scale=0.3)
        scores = (qt @ kt.transpose(-1, -2)) * 0.3
        want_lse = scipy.special.logsumexp(scores.masked_fill(~mask, float("-inf")).numpy(), axis=-1)
        o, lse = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, causal, 0.3, window_left=window,
                                        lib=lib)
        what = f"varlen causal={causal} window={window}"
        assert np.max(np.abs(o - want[0].permute(1, 0, 2).numpy())) < 1e-10, what + ": O"
        assert np.max(np.abs(lse - want_lse[0])) < 1e-10, what + ": LSE"


def pin_varlen_sequences_are_independent(lib):
    """Changing one sequence's tokens changes no other sequence's result."""
    q, k, v, cu_q, cu_k = _varlen_case(32, [6, 4, 8], [6, 10, 8])
    o1, l1 = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, False, 0.25, lib=lib)
    k2, v2 = k.clone(), v.clone()
    k2[cu_k[1]:cu_k[2]] = bf16(np.full(k2[cu_k[1]:cu_k[2]].shape, 1.5))
    v2[cu_k[1]:cu_k[2]] = bf16(np.full(v2[cu_k[1]:cu_k[2]].shape, -0.5))
    o2, l2 = oracle.attn_fwd_varlen(q, k2, v2, cu_q, cu_k, False, 0.25, lib=lib)
    other = np.r_[cu_q[0]:cu_q[1], cu_q[2]:cu_q[3]]
    assert np.array_equal(o1[other], o2[other]) and np.array_equal(l1[:, other], l2[:, other])
    # Identical V rows in the changed sequence: its outputs are -0.5 (the
    # weights sum to 1 up to FP64 rounding).
    assert np.all(np.abs(o2[cu_q[1]:cu_q[2]] + 0.5) < 1e-14)


# ------------------------------------------------------------------ backward
def _torch_grads(q, k, v, dout, scale, mask=None):
    """dQ, dK, dV from torch's float64 autograd of its SDPA (an independent
    library routine), for L = sum(O * dO); layouts as the oracle's."""
    qt = q.double().permute(0, 2, 1, 3).requires_grad_()
    kt = k.double().permute(0, 2, 1, 3).requires_grad_()
    vt = v.double().permute(0, 2, 1, 3).requires_grad_()
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale,
                                                         enable_gqa=True)
    (o * dout.double().permute(0, 2, 1, 3)).sum().backward()
    return tuple(t.grad.permute(0, 2, 1, 3).numpy() for t in (qt, kt, vt))


def pin_bwd_torch_autograd_f64(lib):
    """Backward = torch float64 autograd of SDPA: MHA and GQA, non-causal,
    bottom-right causal and a sliding window (as explicit boolean masks)."""
    for (hq, hkv, sq, sk, causal, w, seed) in [(4, 4, 21, 21, False, -1, 41),
                                              (4, 2, 19, 30, True, -1, 42),
                                              (6, 3, 25, 25, True, 5, 43),
                                              (2, 1, 1, 17, True, -1, 44)]:
        q, k, v = make_qkv(2, hq, hkv, sq, sk, seed=seed, d=16)
        dout = make_qkv(2, hq, hkv, sq, sk, seed=seed + 100, d=16)[0]
        mask = None
        if causal:
            i = torch.arange(sq)[:, None]
            j = torch.arange(sk)[None, :]
            mask = j <= i + (sk - sq)
            if w >= 0:
                mask &= j >= i + (sk - sq) - w
        got = oracle.attn_bwd(q, k, v, dout, causal, 0.35, window_left=w, lib=lib)
        want = _torch_grads(q, k, v, dout, 0.35, mask)
        for name, g, t in zip(("dQ", "dK", "dV"), got, want):
            assert np.max(np.abs(g - t)) < 1e-11, f"{name} vs torch autograd ({hq}/{hkv})"


def pin_bwd_finite_differences(lib):
    """Central differences of the (pinned) forward oracle: for
    L = sum(O * dO), dL/dx ~ (L(x + e) - L(x - e)) / 2e.  Inputs and steps sit
    on a 2^-6 grid, so x +- e stays exact in BF16."""
    rng = np.random.default_rng(45)
    b, hq, hkv, sq, sk, d, scale = 1, 2, 1, 9, 11, 8, 0.4
    e = 2.0 ** -6
    base = [grid_values(rng, shp, -1.0, 1.0, e) for shp in
            ((b, sq, hq, d), (b, sk, hkv, d), (b, sk, hkv, d))]
    dout = grid_values(rng, (b, sq, hq, d), -1.0, 1.0, e)

    def loss(arrs, causal):
        o, _, _ = run(lib, bf16(arrs[0]), bf16(arrs[1]), bf16(arrs[2]), causal, scale)
        return float(np.sum(o.transpose(0, 2, 1, 3) * dout))

    for causal in (False, True):
        grads = oracle.attn_bwd(bf16(base[0]), bf16(base[1]), bf16(base[2]), bf16(dout), causal,
                                scale, lib=lib)
        for which in range(3):
            for _ in range(4):
                idx = tuple(int(rng.integers(0, n)) for n in base[which].shape)
                plus = [a.copy() for a in base]
                minus = [a.copy() for a in base]
                plus[which][idx] += e
                minus[which][idx] -= e
                fd = (loss(plus, causal) - loss(minus, causal)) / (2 * e)
                g = grads[which][idx]
                assert abs(fd - g) <= 2e-4 + 2e-3 * abs(g), f"finite difference, input {which}"


def pin_bwd_invariants(lib):
    """Facts of the chain rule that need no second implementation: each row
    of dS sums to 0, so the dK rows of a key/value head sum to 0; each row of
    P sums to 1, so the dV rows sum to the sum of the group's dO rows; with
    identical V rows dP is constant along a row, so dS = 0 and dQ = dK = 0."""
    q, k, v = make_qkv(2, 4, 2, 23, 23, seed=46, d=8)
    dout = make_qkv(2, 4, 2, 23, 23, seed=47, d=8)[0]
    for causal in (False, True):
        dq, dk, dv = oracle.attn_bwd(q, k, v, dout, causal, 0.5, lib=lib)
        assert np.max(np.abs(dk.sum(axis=1))) < 1e-12, "dK rows do not sum to 0"
        do = dout.double().numpy()
        want = do.reshape(2, 23, 2, 2, 8).sum(axis=(1, 3))          # [b, kv head, d]
        assert np.max(np.abs(dv.sum(axis=1) - want)) < 1e-12, "dV rows do not sum to sum dO"
    rng = np.random.default_rng(48)
    vrow = grid_values(rng, (2, 1, 2, 8))
    v_same = bf16(np.broadcast_to(vrow, (2, 23, 2, 8)).copy())
    dq, dk, dv = oracle.attn_bwd(q, k, v_same, dout, True, 0.5, lib=lib)
    assert np.max(np.abs(dq)) < 1e-12 and np.max(np.abs(dk)) < 1e-12, "identical V rows"
    # Causal, square: the last key is seen by the last row only.
    _, _, p = run(lib, q, k, v, True, 0.5, want_p=True)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, True, 0.5, lib=lib)
    want_v = sum(p[:, h, 22, 22][:, None] * do[:, 22, h] for h in (2, 3))   # kv head 1
    assert np.max(np.abs(dv[:, 22, 1] - want_v)) < 1e-12, "causal last key"


# ------------------------------------------------------------------ FP8 inputs
def _fp8_case(seed, b=2, hq=4, hkv=2, s_q=19, s_k=23, d=16):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(b, s_q, hq, d, generator=g).to(torch.float8_e4m3fn)
    k = torch.randn(b, s_k, hkv, d, generator=g).to(torch.float8_e4m3fn)
    v = torch.randn(b, s_k, hkv, d, generator=g).to(torch.float8_e4m3fn)
    return q, k, v


def pin_e4m3_decode_all_codes(lib):
    """The oracle's E4M3 decoding of all 256 codes equals torch's float8_e4m3fn
    conversion (NaN codes included)."""
    codes = torch.arange(256, dtype=torch.uint8)
    want = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([float(lib.oracle_e4m3_to_double(c)) for c in range(256)])
    assert np.array_equal(np.isnan(want), np.isnan(got)), "E4M3 NaN codes"
    ok = ~np.isnan(want)
    assert np.array_equal(want[ok], got[ok]), "E4M3 values"


def pin_fp8_forward_is_the_forward_of_the_dequantized_inputs(lib):
    """With power-of-two scales every dequantized input is exactly a BF16
    value, so the FP8 forward must equal the (pinned) BF16 forward on those
    values bit for bit; with other scales it must equal torch's float64
    SDPA on the dequantized values."""
    q, k, v = _fp8_case(51)
    for (qs, ks, vs) in [(0.5, 2.0, 0.25), (1.0, 1.0, 1.0)]:
        for causal in (False, True):
            o8, l8 = oracle.attn_fwd_fp8(q, k, v, qs, ks, vs, causal, 0.3, lib=lib)
            qb = bf16(q.to(torch.float64).numpy() * qs)
            kb = bf16(k.to(torch.float64).numpy() * ks)
            vb = bf16(v.to(torch.float64).numpy() * vs)
            o, l, _ = run(lib, qb, kb, vb, causal, 0.3)
            assert np.array_equal(o8, o) and np.array_equal(l8, l), "FP8 vs BF16 forward"
    qs, ks, vs = 0.37, 1.9, 0.61
    o8, l8 = oracle.attn_fwd_fp8(q, k, v, qs, ks, vs, True, 0.3, lib=lib)
    qt = (q.to(torch.float64) * qs).permute(0, 2, 1, 3)
    kt = (k.to(torch.float64) * ks).permute(0, 2, 1, 3).repeat_interleave(2, 1)
    vt = (v.to(torch.float64) * vs).permute(0, 2, 1, 3).repeat_interleave(2, 1)
    mask = torch.ones(19, 23, dtype=torch.bool).tril(4)
    want = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=0.3)
    assert np.max(np.abs(o8 - want.numpy())) < 1e-12, "FP8 forward vs torch SDPA"


ALL_PINS = [
    pin_rows_sum_to_one, pin_identical_v_rows, pin_zero_query, pin_causal_row0,
    pin_causal_rectangular_is_square_suffix, pin_causal_single_query_sees_every_key,
    pin_window_covering_every_key_is_causal, pin_window_zero_keeps_the_diagonal_key,
    pin_window_row_is_attention_over_its_keys, pin_key_split_merge,
    pin_key_shift, pin_value_affine, pin_key_permutation, pin_gqa_equals_repeated_mha,
    pin_torch_sdpa_f64, pin_golden_closed_forms, pin_row_subset,
    pin_varlen_matches_block_diagonal_sdpa, pin_varlen_sequences_are_independent,
    pin_bwd_torch_autograd_f64, pin_bwd_finite_differences, pin_bwd_invariants,
    pin_e4m3_decode_all_codes, pin_fp8_forward_is_the_forward_of_the_dequantized_inputs,
]


def failing_pins(lib) -> list[str]:
    """Names of the pins the given oracle library fails (errors count as fails)."""
    bad = []
    for pin in ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(lib)
        except Exception as exc:  # noqa: BLE001 - any failure is a catch
            bad.append(f"{pin.__name__}: {type(exc).__name__}")
    return bad

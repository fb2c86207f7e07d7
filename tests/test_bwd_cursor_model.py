"""CPU model of the backward dK/dV kernel's work items (no GPU needed).

`Cursor::decode` in csrc/attn_bwd_kernel.cuh (namespace dkdv) maps item t to
(batch, key/value head, key block) inside sections of heads, and gives the
query blocks that see the key block: lo from the causal diagonal (a floor
division by 128 of kb * 128 - (s_k - s_q)) and hi from the sliding window.
Items with no query block (nq = 0) are skipped by the main loop, and
`zero_unseen_key_blocks` writes their dK and dV rows as zeros instead.

This model restates that decode (C++ arithmetic: >> floors negative values)
and checks, over rectangular shapes, windows and section sizes, that:
every (batch, head, key block) is exactly one item; nq = 0 exactly when no
query row sees any key of the block (so zeros are the right gradient there
and every other block goes through the main loop); and the skipped blocks
are a prefix of the key sequence (the keys before the first query's window).
"""
from __future__ import annotations

import itertools

import pytest


def decode(t, batch, h_kv, n_kb, n_qb, section, off, window):
    bg_count = batch * h_kv
    per_sec = section * n_kb
    sec = t // per_sec
    in_sec = min(section, bg_count - sec * section)
    r = t - sec * per_sec
    kb = r // in_sec
    bg = sec * section + (r - kb * in_sec)
    b, g = divmod(bg, h_kv)
    lo = max(0, (kb * 128 - off) >> 7)
    hi = n_qb
    if window >= 0:
        last = kb * 128 + 127 + window - off
        hi = min(hi, (last >> 7) + 1)
    return b, g, kb, lo, max(0, hi - lo)


def seen_by_some_query(kb, s_q, s_k, window):
    off = s_k - s_q
    for j in range(kb * 128, min(kb * 128 + 128, s_k)):
        # query i sees key j iff i + off - window <= j <= i + off (window >= 0)
        i_lo = max(0, j - off)
        i_hi = s_q - 1 if window < 0 else min(s_q - 1, j - off + window)
        if i_lo <= i_hi:
            return True
    return False


SHAPES = [(s_q, s_k) for s_q, s_k in itertools.product([1, 100, 128, 129, 383],
                                                        [128, 384, 700, 1025]) if s_q <= s_k]


@pytest.mark.parametrize("window", [-1, 0, 37, 128, 130, 500])
def test_dkdv_items_and_unseen_key_blocks(window):
    for s_q, s_k in SHAPES:
        check_shape(s_q, s_k, window)


def check_shape(s_q, s_k, window):
    off = s_k - s_q
    w = -1 if window >= s_k else window  # the host's rule: a window of s_k keys is none
    n_qb, n_kb = -(-s_q // 128), -(-s_k // 128)
    for batch, h_kv in [(1, 1), (2, 3), (3, 4)]:
        n_items = batch * h_kv * n_kb
        for section in sorted({batch * h_kv, min(4, batch * h_kv)}):
            items = [decode(t, batch, h_kv, n_kb, n_qb, section, off, w) for t in range(n_items)]
            assert sorted((b, g, kb) for b, g, kb, _, _ in items) == [
                (b, g, kb) for b in range(batch) for g in range(h_kv) for kb in range(n_kb)]
            skipped = set()
            for b, g, kb, lo, nq in items:
                assert (nq > 0) == seen_by_some_query(kb, s_q, s_k, w), (b, g, kb, lo, nq)
                if nq == 0:
                    skipped.add(kb)
                else:
                    assert 0 <= lo and lo + nq <= n_qb
            assert skipped == set(range(len(skipped))), "skipped blocks are not a prefix"
            if w < 0:
                assert not skipped, "without a window every key block is seen"

"""CPU model of how the persistent forward kernel deals causal work items to
its CTAs.

Items are (query-block pair) work units ordered longest first; the kernel
deals them to the G persistent CTAs in rounds of G, in a snake order (round
k: CTA c takes item kG + c when k is even and kG + G - 1 - c when k is
odd).  Causal pair p of a square problem visits 2p + 1 and 2p + 2 key blocks;
each pair also pays a fixed boundary cost (about 8 half-steps of work: the
TMA store of O, the next pair's Q load).  The model sums each CTA's work and
compares the busiest CTA with the mean: the snake deal of one longest-first
order balances the causal MHA workloads to within a few percent, where a
plain grid stride (CTA c takes items c, c + G, ...) leaves the busiest CTA
10-14 % over the mean.
"""
from __future__ import annotations

import pytest

G = 148  # persistent CTAs: one per SM


def causal_items(batch, h_q, s):
    """Work of each item in the kernel's causal order: pair descending, then
    (batch, head)."""
    n_qb = (s + 127) // 128
    n_pairs = (n_qb + 1) // 2
    items = []
    for pair in reversed(range(n_pairs)):
        qb0 = 2 * pair
        n0 = qb0 + 1
        n1 = qb0 + 2 if qb0 + 1 < n_qb else 0
        items += [n0 + n1 + 8] * (batch * h_q)
    return items


def busiest_over_mean(items, snake):
    load = [0] * G
    for t, w in enumerate(items):
        k, pos = divmod(t, G)
        c = G - 1 - pos if (snake and k % 2) else pos
        load[c] += w
    return max(load) / (sum(load) / G)


@pytest.mark.parametrize("batch,h_q,s", [(8, 16, 4096), (4, 16, 8192), (2, 16, 16384),
                                         (1, 16, 32768)])
def test_snake_deal_balances_causal_mha(batch, h_q, s):
    items = causal_items(batch, h_q, s)
    snake = busiest_over_mean(items, True)
    stride = busiest_over_mean(items, False)
    assert snake <= 1.015, snake
    assert stride >= 1.05, stride


def test_snake_deal_of_equal_items_is_the_grid_stride():
    items = [10] * (3 * G + 17)
    assert busiest_over_mean(items, True) == busiest_over_mean(items, False)

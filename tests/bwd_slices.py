"""The FP64 oracle's backward of one (batch, key/value head) group,
assembled from oracle calls on slices of query rows (test infrastructure).

Each query row's P and dS depend only on that row (its own softmax over all
the keys it sees), so the rows of dQ come out of the slice that holds them
and dK, dV are the sums of the slices' contributions.  A causal slice of
rows [a, a + m) is given the keys [0, a + m + s_k - s_q): the oracle aligns
the mask to the bottom-right corner, so every row keeps exactly the keys it
sees in the whole problem.  Slices of 128 rows keep the oracle's score
matrices in cache, and the slices run in threads (the oracle's calls
release the interpreter lock).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

import oracle

ROWS = 128


def oracle_group(q, k, v, dout, b, g, group, causal, scale, rows=ROWS):
    """FP64 dQ of the group's query heads [s_q, group, d] and dK, dV of key/
    value head g [s_k, d], from oracle calls on query slices of `rows` rows."""
    qb, kb, vb, ob = (oracle._as_bits(t) for t in (q, k, v, dout))
    s_q, s_k, d = qb.shape[1], kb.shape[1], qb.shape[3]
    off = s_k - s_q
    lib = oracle.load()
    kg = np.ascontiguousarray(kb[b:b + 1, :, g:g + 1])
    vg = np.ascontiguousarray(vb[b:b + 1, :, g:g + 1])

    def piece(job):
        hl, a = job
        h = g * group + hl
        e = min(s_k, a + rows + off) if causal else s_k
        dq, dk, dv = oracle.attn_bwd(np.ascontiguousarray(qb[b:b + 1, a:a + rows, h:h + 1]),
                                     np.ascontiguousarray(kg[:, :e]),
                                     np.ascontiguousarray(vg[:, :e]),
                                     np.ascontiguousarray(ob[b:b + 1, a:a + rows, h:h + 1]),
                                     causal, scale, lib=lib)
        return hl, a, e, dq[0, :, 0], dk[0, :, 0], dv[0, :, 0]

    jobs = [(hl, a) for hl in range(group) for a in range(0, s_q, rows)]
    dq = np.zeros((s_q, group, d))
    dk = np.zeros((s_k, d))
    dv = np.zeros((s_k, d))
    with ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        for hl, a, e, pq, pk, pv in ex.map(piece, jobs):
            dq[a:a + pq.shape[0], hl] = pq
            dk[:e] += pk
            dv[:e] += pv
    return dq, dk, dv

"""Seeded synthetic workloads for the attention forward.

This module holds only shapes, seeds and random draws -- none of the
method's arithmetic -- so the CUDA path and the FP64 oracle can be fed the
same bits without sharing any code.

Shapes follow the workloads the pages measure on: head dim 128, 16 query
heads, BF16, sequence 4K-32K with the batch shrinking as the sequence grows
(intelliparadigm.com AVO page, section 1 note), and batch 8 / 16 heads /
sequence 2048 with grouped or single key/value heads (rkmt.cn page,
section 4.1).  Every tensor is drawn as N(0, 1) in FP32 from a CPU
``torch.Generator`` and rounded to BF16, so the bits are identical on every
machine.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

HEAD_DIM = 128


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    h_q: int
    h_kv: int
    seq: int
    seed: int
    k_scale: float = 1.0   # K drawn as k_scale * N(0,1) before rounding
    sampled: bool = False  # parity on sampled query rows (long sequences)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(HEAD_DIM)

    def flops(self, causal: bool) -> float:
        """4 * b * h_q * s_q * s_k * d, halved for causal."""
        f = 4.0 * self.batch * self.h_q * self.seq * self.seq * HEAD_DIM
        return f / 2 if causal else f

    def input_bytes(self) -> int:
        """Q, K and V (BF16)."""
        return 2 * HEAD_DIM * (self.batch * self.seq * self.h_q + 2 * self.batch * self.seq * self.h_kv)

    def algorithmic_bytes(self) -> int:
        """Q, K, V and O moved once (BF16) plus the FP32 LSE."""
        q = self.batch * self.seq * self.h_q * HEAD_DIM * 2
        kv = 2 * self.batch * self.seq * self.h_kv * HEAD_DIM * 2
        lse = self.batch * self.h_q * self.seq * 4
        return 2 * q + kv + lse


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_b1_h2_s256", 1, 2, 2, 256, 1001),
        Workload("mha_b8_h16_s4096", 8, 16, 16, 4096, 1002),
        Workload("mha_b4_h16_s8192", 4, 16, 16, 8192, 1003, sampled=True),
        Workload("mha_b2_h16_s16384", 2, 16, 16, 16384, 1013, sampled=True),
        Workload("mha_b1_h16_s32768_k3", 1, 16, 16, 32768, 1004, k_scale=3.0, sampled=True),
        Workload("gqa_b8_h16_kv2_s2048", 8, 16, 2, 2048, 1005),
        Workload("mqa_b8_h16_kv1_s2048", 8, 16, 1, 2048, 1006),
    ]
}


def make_qkv(batch: int, h_q: int, h_kv: int, s_q: int, s_k: int, seed: int,
             d: int = HEAD_DIM, k_scale: float = 1.0, dist: str = "normal"):
    """Q [b, s_q, h_q, d], K/V [b, s_k, h_kv, d] as BF16 CPU tensors.

    Draw order is Q, K, V from one generator seeded with ``seed``.
    ``dist='normal'`` draws N(0,1); ``dist='uniform'`` draws U(-1,1).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)

    def draw(shape):
        if dist == "normal":
            return torch.randn(shape, generator=g, dtype=torch.float32)
        if dist == "uniform":
            return torch.rand(shape, generator=g, dtype=torch.float32) * 2 - 1
        raise ValueError(dist)

    q = draw((batch, s_q, h_q, d)).to(torch.bfloat16)
    k = (draw((batch, s_k, h_kv, d)) * k_scale).to(torch.bfloat16)
    v = draw((batch, s_k, h_kv, d)).to(torch.bfloat16)
    return q, k, v


def workload_qkv(w: Workload):
    return make_qkv(w.batch, w.h_q, w.h_kv, w.seq, w.seq, w.seed, k_scale=w.k_scale)


# Rows every sample keeps: first rows, both sides of the first tile edges,
# and the last row.
EDGE_ROWS = (0, 1, 127, 128, 255, 256)


def sample_rows(batch: int, h_q: int, s_q: int, n: int, seed: int,
                include_edges: bool = True) -> np.ndarray:
    """Seeded per-(batch, head) sample of ``n`` distinct query rows, sorted.

    With ``include_edges`` the sample always contains the edge rows (0, 1,
    127, 128, 255, 256, s_q-1 where they exist; ``n`` is raised to hold them).
    Returns int32 [batch, h_q, n'] with n' = min(n, s_q).
    """
    fixed = sorted({r for r in EDGE_ROWS if r < s_q} | {s_q - 1}) if include_edges else []
    n = min(max(n, len(fixed)), s_q)
    rng = np.random.default_rng(seed)
    out = np.empty((batch, h_q, n), dtype=np.int32)
    pool = np.setdiff1d(np.arange(s_q), np.array(fixed, dtype=np.int64))
    for b in range(batch):
        for h in range(h_q):
            if n >= s_q:
                out[b, h] = np.arange(s_q, dtype=np.int32)
                continue
            extra = rng.choice(pool, size=n - len(fixed), replace=False)
            out[b, h] = np.sort(np.concatenate([np.array(fixed, dtype=np.int64), extra])).astype(np.int32)
    return out


def make_qkv_fp8(batch: int, h_q: int, h_kv: int, s_q: int, s_k: int, seed: int,
                 d: int = HEAD_DIM, k_scale: float = 1.0):
    """FP8 E4M3 Q, K, V with per-tensor scales: the same N(0, 1) draws as
    :func:`make_qkv` (FP32, before any rounding), each tensor divided by its
    scale amax / 448 and rounded to E4M3 (torch's conversion).  Returns
    (q8, k8, v8, q_scale, k_scale, v_scale): the inputs stand for scale * x8."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn((batch, s_q, h_q, d), generator=g, dtype=torch.float32)
    k = torch.randn((batch, s_k, h_kv, d), generator=g, dtype=torch.float32) * k_scale
    v = torch.randn((batch, s_k, h_kv, d), generator=g, dtype=torch.float32)
    out = []
    scales = []
    for t in (q, k, v):
        sc = float(t.abs().max()) / 448.0
        out.append((t / sc).to(torch.float8_e4m3fn))
        scales.append(sc)
    return (*out, *scales)

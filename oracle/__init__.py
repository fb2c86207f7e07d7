"""FP64 CPU oracle for the scaled dot-product attention forward.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import this package; the
product package (``scaled_dot_product_10_b200``) never does, and the oracle
never imports the product.  The arithmetic lives in ``attn_oracle.c`` (plain
C, FP64): it materialises S, masks it, takes the row max, exponentiates,
normalises and multiplies by V, exactly as the definition
``softmax(Q K^T / sqrt(d_k)) V`` on the rkmt.cn page (section 1) states.

This module only marshals numpy arrays into that C function.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math: the FP64
    arithmetic keeps IEEE semantics and program order)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-fno-fast-math", "-ffp-contract=off", src, "-o", out, "-lm"]
        subprocess.run(cmd, check=True)
    return out


def load(path: str | None = None):
    """Load (building if needed) the oracle shared library."""
    global _lib
    if path is not None:
        lib = ctypes.CDLL(path)
    else:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
    lib.oracle_attn_fwd_f64.restype = ctypes.c_int
    lib.oracle_attn_fwd_f64.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_double,
        ctypes.c_void_p, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
    ]
    lib.oracle_attn_bwd_f64.restype = ctypes.c_int
    lib.oracle_attn_bwd_f64.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_double,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
    ]
    lib.oracle_attn_fwd_fp8_f64.restype = ctypes.c_int
    lib.oracle_attn_fwd_fp8_f64.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_double, ctypes.c_double, ctypes.c_double,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_double,
        ctypes.c_void_p, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
    ]
    lib.oracle_e4m3_to_double.restype = ctypes.c_double
    lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
    lib.oracle_num_threads.restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def num_threads() -> int:
    return int(load().oracle_num_threads())


def _as_bits(x) -> np.ndarray:
    """Accept a torch bf16 tensor or a numpy uint16 array of bf16 bits."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy inputs must be uint16 arrays of bf16 bits")
        return np.ascontiguousarray(x)
    import torch  # local: only for the tensor -> bits view
    if x.dtype != torch.bfloat16:
        raise TypeError("torch inputs must be bfloat16")
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def attn_fwd(q, k, v, causal: bool, scale: float, rows=None, want_p: bool = False, lib=None,
             window_left: int = -1):
    """Run the oracle.

    q: [batch, s_q, h_q, d] bf16 (torch tensor or uint16 bits);
    k, v: [batch, s_k, h_kv, d].
    rows: None (every query row) or an int array [batch, h_q, n_rows] of the
    query indices to evaluate per (batch, head).
    window_left: -1 (none) or, with causal, the sliding window: row i sees
    keys i + s_k - s_q - window_left .. i + s_k - s_q.

    Returns (o, lse, p): o [batch, h_q, n_rows, d] float64,
    lse [batch, h_q, n_rows] float64 (natural log), p [batch, h_q, n_rows, s_k]
    float64 or None.
    """
    qb, kb, vb = _as_bits(q), _as_bits(k), _as_bits(v)
    batch, s_q, h_q, d = qb.shape
    bk, s_k, h_kv, dk = kb.shape
    if vb.shape != kb.shape or bk != batch or dk != d:
        raise ValueError("shape mismatch between q, k and v")
    if rows is None:
        n_rows = s_q
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        if rows_arr.ndim != 3 or rows_arr.shape[:2] != (batch, h_q):
            raise ValueError("rows must have shape [batch, h_q, n_rows]")
        n_rows = rows_arr.shape[2]
    o = np.zeros((batch, h_q, n_rows, d), dtype=np.float64)
    lse = np.zeros((batch, h_q, n_rows), dtype=np.float64)
    p = np.zeros((batch, h_q, n_rows, s_k), dtype=np.float64) if want_p else None
    lib = lib or load()
    rc = lib.oracle_attn_fwd_f64(
        qb.ctypes.data, kb.ctypes.data, vb.ctypes.data,
        batch, h_q, h_kv, s_q, s_k, d, int(bool(causal)), int(window_left), float(scale),
        None if rows_arr is None else rows_arr.ctypes.data, n_rows,
        o.ctypes.data, lse.ctypes.data, None if p is None else p.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")
    return o, lse, p


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, causal: bool, scale: float,
                    window_left: int = -1, lib=None):
    """Packed variable-length batch: the definition applied to each sequence
    on its own (attention never crosses sequences).

    q: [total_q, h_q, d] bf16; k, v: [total_k, h_kv, d].  Sequence b holds
    query rows cu_seqlens_q[b] .. cu_seqlens_q[b+1] - 1 and keys
    cu_seqlens_k[b] .. cu_seqlens_k[b+1] - 1; the causal mask (and window)
    is that of a single problem with that sequence's s_q and s_k.  A
    sequence with no query rows contributes nothing; one with query rows but
    no keys is rejected.

    Returns (o [total_q, h_q, d] float64, lse [h_q, total_q] float64).
    """
    qb, kb, vb = _as_bits(q), _as_bits(k), _as_bits(v)
    cu_q = [int(x) for x in np.asarray(cu_seqlens_q).reshape(-1)]
    cu_k = [int(x) for x in np.asarray(cu_seqlens_k).reshape(-1)]
    if len(cu_q) != len(cu_k) or len(cu_q) < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k need batch + 1 entries each")
    total_q, h_q, d = qb.shape
    total_k, h_kv, dk = kb.shape
    if vb.shape != kb.shape or dk != d:
        raise ValueError("shape mismatch between q, k and v")
    if cu_q[0] != 0 or cu_k[0] != 0 or cu_q[-1] != total_q or cu_k[-1] != total_k:
        raise ValueError("cu_seqlens must start at 0 and end at the packed lengths")
    o = np.zeros((total_q, h_q, d), dtype=np.float64)
    lse = np.zeros((h_q, total_q), dtype=np.float64)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        if q1 < q0 or k1 < k0:
            raise ValueError("cu_seqlens must not decrease")
        if q1 == q0:
            continue
        if k1 == k0:
            raise ValueError(f"sequence {b} has query rows but no keys")
        ob, lb, _ = attn_fwd(qb[None, q0:q1], kb[None, k0:k1], vb[None, k0:k1], causal, scale,
                             lib=lib, window_left=window_left)
        o[q0:q1] = ob[0].transpose(1, 0, 2)
        lse[:, q0:q1] = lb[0]
    return o, lse


def attn_bwd(q, k, v, dout, causal: bool, scale: float, window_left: int = -1, lib=None):
    """Gradients of the forward: given dO (the gradient of a loss with
    respect to O), returns (dq, dk, dv) as float64 arrays in the layouts of
    q, k and v ([batch, s, heads, d]).  q, k, v, dout: bf16 (torch tensors
    or uint16 bits), dout shaped like q."""
    qb, kb, vb, ob = _as_bits(q), _as_bits(k), _as_bits(v), _as_bits(dout)
    batch, s_q, h_q, d = qb.shape
    bk, s_k, h_kv, dk_ = kb.shape
    if vb.shape != kb.shape or bk != batch or dk_ != d or ob.shape != qb.shape:
        raise ValueError("shape mismatch between q, k, v and dout")
    dq = np.zeros((batch, s_q, h_q, d), dtype=np.float64)
    dk = np.zeros((batch, s_k, h_kv, d), dtype=np.float64)
    dv = np.zeros((batch, s_k, h_kv, d), dtype=np.float64)
    lib = lib or load()
    rc = lib.oracle_attn_bwd_f64(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, ob.ctypes.data,
                                 batch, h_q, h_kv, s_q, s_k, d, int(bool(causal)),
                                 int(window_left), float(scale), dq.ctypes.data, dk.ctypes.data,
                                 dv.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")
    return dq, dk, dv


def _as_bytes(x) -> np.ndarray:
    """Accept a torch float8_e4m3fn / uint8 tensor or a numpy uint8 array."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint8:
            raise TypeError("numpy FP8 inputs must be uint8 arrays of e4m3 bits")
        return np.ascontiguousarray(x)
    import torch
    t = x.detach().cpu().contiguous()
    if t.dtype not in (torch.float8_e4m3fn, torch.uint8):
        raise TypeError("torch FP8 inputs must be float8_e4m3fn (or uint8 bits)")
    return np.ascontiguousarray(t.view(torch.uint8).numpy())


def e4m3_to_double(bits: int, lib=None) -> float:
    return float((lib or load()).oracle_e4m3_to_double(int(bits)))


def attn_fwd_fp8(q, k, v, q_scale: float, k_scale: float, v_scale: float, causal: bool,
                 scale: float, rows=None, lib=None, window_left: int = -1):
    """The forward on FP8 E4M3 inputs with per-tensor scales (input values are
    scale * e4m3 value).  Shapes and outputs as :func:`attn_fwd`."""
    qb, kb, vb = _as_bytes(q), _as_bytes(k), _as_bytes(v)
    batch, s_q, h_q, d = qb.shape
    bk, s_k, h_kv, dk = kb.shape
    if vb.shape != kb.shape or bk != batch or dk != d:
        raise ValueError("shape mismatch between q, k and v")
    if rows is None:
        n_rows, rows_arr = s_q, None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        if rows_arr.ndim != 3 or rows_arr.shape[:2] != (batch, h_q):
            raise ValueError("rows must have shape [batch, h_q, n_rows]")
        n_rows = rows_arr.shape[2]
    o = np.zeros((batch, h_q, n_rows, d), dtype=np.float64)
    lse = np.zeros((batch, h_q, n_rows), dtype=np.float64)
    lib = lib or load()
    rc = lib.oracle_attn_fwd_fp8_f64(
        qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, float(q_scale), float(k_scale),
        float(v_scale), batch, h_q, h_kv, s_q, s_k, d, int(bool(causal)), int(window_left),
        float(scale), None if rows_arr is None else rows_arr.ctypes.data, n_rows,
        o.ctypes.data, lse.ctypes.data, None)
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")
    return o, lse

"""ctypes binding of the C ABI in ``include/attn_fwd.h``.

Argument marshalling only: every step of the forward runs in the CUDA
library.  Loading fails loudly if the library is missing -- there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import math
import os

ATTN_OK = 0
ATTN_ERR_INVALID = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_ALIGN = 3
ATTN_ERR_CUDA = 4
ATTN_ERR_TIMEOUT = 5
ATTN_ERR_TOO_LARGE = 6
STATIC_STAGING_BYTES = 32 << 20

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libattn_sm100.so"
_lib = None

# (name, restype, argtypes) of every exported entry point.
_P = ctypes.c_void_p
_I = ctypes.c_int
_SIGNATURES = [
    ("attn_fwd", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P]),
    ("attn_fwd_window", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P]),
    ("attn_fwd_varlen", _I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                             _I, ctypes.c_float, _P]),
    ("attn_bwd_workspace_bytes", ctypes.c_size_t, [_I, _I, _I]),
    ("attn_bwd", _I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I,
                      ctypes.c_float, _P, ctypes.c_size_t, _P]),
    ("attn_fwd_fp8", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float,
                          ctypes.c_float, ctypes.c_float, ctypes.c_float, _P]),
    ("attn_fwd_host", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float,
                           _P, ctypes.c_size_t, _P]),
    ("attn_fwd_host_workspace_bytes", ctypes.c_size_t, [_I, _I, _I, _I, _I, _I]),
    ("attn_fwd_host_static", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float,
                                  _P]),
    ("attn_fwd_num_splits", _I, [_I, _I, _I, _I, _I, _I, _I]),
    ("attn_fwd_split_workspace_bytes", ctypes.c_size_t, [_I, _I, _I, _I]),
    ("attn_fwd_split", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I,
                            _P, ctypes.c_size_t, _P]),
    ("attn_fwd_partials_shard", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I,
                                     ctypes.c_float, _P]),
    ("attn_merge_partials", _I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    ("attn_fwd_partials", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float,
                               _P]),
    ("attn_status", _I, [_P]),
    ("attn_strerror", ctypes.c_char_p, [_I]),
    ("attn_set_wait_timeout_ns", _I, [ctypes.c_uint64]),
    ("attn_selftest_wait_timeout", _I, [ctypes.c_uint64, _P]),
    ("attn_last_launch_count", _I, []),
]
EXPORTED = [s[0] for s in _SIGNATURES]


class AttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {attn_strerror(code)} (code {code})")


def library_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def load_library(path: str | None = None):
    """Load the CUDA library (raises OSError if it is not built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or library_path()
    if not os.path.exists(p):
        raise OSError(f"{p} is missing: build it with `python -m scaled_dot_product_10_b200.build`")
    lib = ctypes.CDLL(p)
    for name, res, args in _SIGNATURES:
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def attn_strerror(code: int) -> str:
    return load_library().attn_strerror(int(code)).decode()


def _stream_handle(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _stream_obj(stream, device):
    """The torch stream object the kernels of a call run on."""
    import torch
    if stream is None:
        return torch.cuda.current_stream(device)
    if isinstance(stream, int):
        return torch.cuda.ExternalStream(stream, device=device)
    return stream


def _cuda_device(stream, **tensors):
    """The one CUDA device every tensor of a call is on.  The library
    launches on the calling thread's current device, so each call runs under
    this device (see :func:`_on_device`); a torch stream given for the call
    must belong to it."""
    dev = None
    for name, t in tensors.items():
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the call's other tensors on {dev}")
    sdev = getattr(stream, "device", None)
    if dev is not None and sdev is not None and sdev != dev:
        raise ValueError(f"stream belongs to {sdev}, the tensors to {dev}")
    return dev


def _on_device(dev):
    """Context making ``dev`` the current device for the library call (and
    for the default stream, torch's current stream on that device)."""
    import torch
    return torch.cuda.device(dev)


def _alloc_on(stream, device, fn):
    """Allocate with ``fn()`` on the launch stream, so the caching allocator
    never hands a buffer that a kernel of this call still uses to work queued
    on another stream once the buffer is dropped."""
    import torch
    with torch.cuda.stream(_stream_obj(stream, device)):
        return fn()


def _check_out(t, name, shape, dtype, device):
    """A caller-supplied output must match what the kernel writes: the C side
    can check only null and alignment."""
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}")


def _check_qkv(q, k, v):
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16")
        if t.dim() != 4:
            raise ValueError(f"{name} must be [batch, seq, heads, head_dim]")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    b, s_q, h_q, d = q.shape
    bk, s_k, h_kv, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or bk != b or dk != d:
        raise ValueError("q, k, v shapes disagree")
    return b, s_q, h_q, h_kv, s_k, d


def _out(ref, t, name, shape, dtype, stream):
    """Check a caller-supplied output, or allocate it on the launch stream."""
    if t is None:
        import torch
        return _alloc_on(stream, ref.device,
                         lambda: torch.empty(shape, dtype=dtype, device=ref.device))
    _check_out(t, name, shape, dtype, ref.device)
    return t


def _outputs(q, o, lse, o_shape, lse_shape, stream, o_dtype=None):
    """Check caller-supplied outputs, or allocate them on the launch stream."""
    import torch
    return (_out(q, o, "o", o_shape, o_dtype or torch.bfloat16, stream),
            _out(q, lse, "lse", lse_shape, torch.float32, stream))


def _workspace(ref, workspace, nbytes, stream):
    """A caller's workspace (contiguous, on the inputs' device, at least
    ``nbytes``; the C side checks the size too) or one allocated on the
    launch stream, whose memory is then not reused before the call's kernels
    finish even though it is dropped on return."""
    if workspace is None:
        import torch
        return _alloc_on(stream, ref.device,
                         lambda: torch.empty(nbytes, dtype=torch.uint8, device=ref.device))
    if workspace.device != ref.device or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous tensor on the inputs' device")
    return workspace


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def attn_fwd(q, k, v, causal: bool = False, scale: float | None = None, o=None, lse=None,
             stream=None):
    """O, LSE = attention forward on CUDA tensors [batch, seq, heads, 128] (BF16).

    Returns (o [b, s_q, h_q, 128] BF16, lse [b, h_q, s_q] FP32).  Asynchronous
    on ``stream`` (default: torch's current stream on the tensors' device).
    """
    b, s_q, h_q, h_kv, s_k, d = _check_qkv(q, k, v)
    dev = _cuda_device(stream, q=q, k=k, v=v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with _on_device(dev):
        o, lse = _outputs(q, o, lse, (b, s_q, h_q, d), (b, h_q, s_q), stream)
        rc = load_library().attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                     lse.data_ptr(), b, h_q, h_kv, s_q, s_k, d,
                                     int(bool(causal)), float(scale), _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd")
    return o, lse


def attn_fwd_window(q, k, v, window_left: int, scale: float | None = None, o=None, lse=None,
                    stream=None):
    """Causal attention where query row i sees only keys
    i + s_k - s_q - window_left .. i + s_k - s_q.  Returns (o, lse) as
    :func:`attn_fwd`."""
    b, s_q, h_q, h_kv, s_k, d = _check_qkv(q, k, v)
    dev = _cuda_device(stream, q=q, k=k, v=v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with _on_device(dev):
        o, lse = _outputs(q, o, lse, (b, s_q, h_q, d), (b, h_q, s_q), stream)
        rc = load_library().attn_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                            o.data_ptr(), lse.data_ptr(), b, h_q, h_kv, s_q,
                                            s_k, d, int(window_left), float(scale),
                                            _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_window")
    return o, lse


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                    causal: bool = False, scale: float | None = None, window_left: int = -1,
                    o=None, lse=None, stream=None):
    """Packed variable-length batch: q [total_q, h_q, 128], k/v
    [total_k, h_kv, 128] (BF16, CUDA), cu_seqlens_* int32 CUDA tensors
    [batch + 1].  Returns (o [total_q, h_q, 128] BF16, lse [h_q, total_q]
    FP32)."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or t.dim() != 3 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{name} must be a contiguous CUDA bfloat16 [tokens, heads, dim]")
    for name, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if t.dtype != torch.int32 or t.dim() != 1 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{name} must be a contiguous CUDA int32 vector")
    dev = _cuda_device(stream, q=q, k=k, v=v, cu_seqlens_q=cu_seqlens_q,
                       cu_seqlens_k=cu_seqlens_k)
    total_q, h_q, d = q.shape
    total_k, h_kv, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or dk != d:
        raise ValueError("q, k, v shapes disagree")
    batch = cu_seqlens_q.numel() - 1
    if cu_seqlens_k.numel() != batch + 1 or batch < 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k need batch + 1 entries")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with _on_device(dev):
        o, lse = _outputs(q, o, lse, (total_q, h_q, d), (h_q, total_q), stream)
        rc = load_library().attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                            o.data_ptr(), lse.data_ptr(),
                                            cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(),
                                            batch, int(max_seqlen_q), int(max_seqlen_k),
                                            total_q, total_k, h_q, h_kv, d, int(bool(causal)),
                                            int(window_left), float(scale),
                                            _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_varlen")
    return o, lse


def bwd_workspace_bytes(b, h_q, s_q) -> int:
    return int(load_library().attn_bwd_workspace_bytes(b, h_q, s_q))


def attn_bwd(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
             window_left: int = -1, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients of the forward: (dq, dk, dv) BF16 in the layouts of q, k, v,
    from the forward's o [b, s_q, h_q, 128] and lse [b, h_q, s_q] and the
    incoming gradient dout (shaped like o).  Three launches on ``stream``."""
    import torch
    b, s_q, h_q, h_kv, s_k, d = _check_qkv(q, k, v)
    dev = _cuda_device(stream, q=q, k=k, v=v)
    _check_out(o, "o", (b, s_q, h_q, d), torch.bfloat16, dev)
    _check_out(dout, "dout", (b, s_q, h_q, d), torch.bfloat16, dev)
    _check_out(lse, "lse", (b, h_q, s_q), torch.float32, dev)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with _on_device(dev):
        dq = _out(q, dq, "dq", (b, s_q, h_q, d), torch.bfloat16, stream)
        dk = _out(q, dk, "dk", (b, s_k, h_kv, d), torch.bfloat16, stream)
        dv = _out(q, dv, "dv", (b, s_k, h_kv, d), torch.bfloat16, stream)
        workspace = _workspace(q, workspace, bwd_workspace_bytes(b, h_q, s_q), stream)
        rc = load_library().attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                     dout.data_ptr(), lse.data_ptr(), dq.data_ptr(),
                                     dk.data_ptr(), dv.data_ptr(), b, h_q, h_kv, s_q, s_k, d,
                                     int(bool(causal)), int(window_left), float(scale),
                                     workspace.data_ptr(), _nbytes(workspace),
                                     _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_bwd")
    return dq, dk, dv


def attn_fwd_fp8(q, k, v, q_scale: float, k_scale: float, v_scale: float, causal: bool = False,
                 scale: float | None = None, o=None, lse=None, stream=None):
    """Forward on FP8 E4M3 CUDA tensors (torch.float8_e4m3fn) [batch, seq,
    heads, 128] standing for q_scale * q, k_scale * k, v_scale * v.  Returns
    (o BF16 [b, s_q, h_q, 128], lse FP32 [b, h_q, s_q])."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.float8_e4m3fn or t.dim() != 4 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{name} must be a contiguous CUDA float8_e4m3fn [b, s, h, d]")
    dev = _cuda_device(stream, q=q, k=k, v=v)
    b, s_q, h_q, d = q.shape
    bk, s_k, h_kv, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or bk != b or dk != d:
        raise ValueError("q, k, v shapes disagree")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with _on_device(dev):
        o, lse = _outputs(q, o, lse, (b, s_q, h_q, d), (b, h_q, s_q), stream)
        rc = load_library().attn_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                         lse.data_ptr(), b, h_q, h_kv, s_q, s_k, d,
                                         int(bool(causal)), float(scale), float(q_scale),
                                         float(k_scale), float(v_scale), _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_fp8")
    return o, lse


def num_splits(b, h_q, h_kv, s_q, s_k, causal=False, d=128) -> int:
    """Key-range count the library picks for these sizes on the current device."""
    return int(load_library().attn_fwd_num_splits(b, h_q, h_kv, s_q, s_k, d, int(bool(causal))))


def split_workspace_bytes(b, h_q, s_q, n_splits) -> int:
    return int(load_library().attn_fwd_split_workspace_bytes(b, h_q, s_q, n_splits))


def attn_fwd_split(q, k, v, causal: bool = False, scale: float | None = None,
                   n_splits: int | None = None, o=None, lse=None, workspace=None, stream=None):
    """attn_fwd through ``n_splits`` key ranges and a merge (two launches).
    ``n_splits`` None: the library's choice (:func:`num_splits`).  The
    partials go to ``workspace`` (a CUDA uint8 tensor of at least
    :func:`split_workspace_bytes` bytes; allocated here if None)."""
    b, s_q, h_q, h_kv, s_k, d = _check_qkv(q, k, v)
    dev = _cuda_device(stream, q=q, k=k, v=v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with _on_device(dev):
        if n_splits is None:
            n_splits = max(1, num_splits(b, h_q, h_kv, s_q, s_k, causal, d))
        o, lse = _outputs(q, o, lse, (b, s_q, h_q, d), (b, h_q, s_q), stream)
        workspace = _workspace(q, workspace, split_workspace_bytes(b, h_q, s_q, n_splits), stream)
        rc = load_library().attn_fwd_split(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                           o.data_ptr(), lse.data_ptr(), b, h_q, h_kv, s_q, s_k,
                                           d, int(bool(causal)), float(scale), int(n_splits),
                                           workspace.data_ptr(), _nbytes(workspace),
                                           _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_split")
    return o, lse


def attn_fwd_partials(q, k, v, causal: bool = False, scale: float | None = None, o_part=None,
                      lse_part=None, stream=None):
    """The unmerged partial of the keys given: O_r FP32 [b, h_q, s_q, 128]
    (normalised over these keys) and LSE_r FP32 [b, h_q, s_q]."""
    import torch
    b, s_q, h_q, h_kv, s_k, d = _check_qkv(q, k, v)
    dev = _cuda_device(stream, q=q, k=k, v=v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with _on_device(dev):
        o_part, lse_part = _outputs(q, o_part, lse_part, (b, h_q, s_q, d), (b, h_q, s_q),
                                    stream, o_dtype=torch.float32)
        rc = load_library().attn_fwd_partials(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                              o_part.data_ptr(), lse_part.data_ptr(), b, h_q,
                                              h_kv, s_q, s_k, d, int(bool(causal)),
                                              float(scale), _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_partials")
    return o_part, lse_part


def shard_diag_offset(s_k_total: int, s_q: int, key_offset: int) -> int:
    """Causal diagonal of a key shard at global key ``key_offset`` when the
    s_q queries are the last s_q positions of ``s_k_total`` keys."""
    return int(s_k_total) - int(s_q) - int(key_offset)


def attn_fwd_partials_shard(q, k, v, causal: bool = False, scale: float | None = None,
                            diag_offset: int | None = None, o_part=None, lse_part=None,
                            stream=None):
    """The unmerged partial of a key shard (see :func:`attn_fwd_partials`);
    with ``causal`` query row i sees shard key j iff j <= i + diag_offset
    (default: s_k - s_q, the whole-problem mask).  Rows that see no key of
    the shard get O_r = 0 and LSE_r = -inf."""
    import torch
    b, s_q, h_q, h_kv, s_k, d = _check_qkv(q, k, v)
    dev = _cuda_device(stream, q=q, k=k, v=v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if diag_offset is None:
        diag_offset = s_k - s_q
    with _on_device(dev):
        o_part, lse_part = _outputs(q, o_part, lse_part, (b, h_q, s_q, d), (b, h_q, s_q),
                                    stream, o_dtype=torch.float32)
        rc = load_library().attn_fwd_partials_shard(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                    o_part.data_ptr(), lse_part.data_ptr(), b,
                                                    h_q, h_kv, s_q, s_k, d, int(bool(causal)),
                                                    int(diag_offset), float(scale),
                                                    _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_partials_shard")
    return o_part, lse_part


def merge_partials(o_parts, lse_parts, o=None, lse=None, stream=None):
    """Merge per-key-range partials: ``o_parts`` FP32 [n, b, h_q, s_q, 128]
    (each normalised over its own keys), ``lse_parts`` FP32 [n, b, h_q, s_q]
    -> O BF16 [b, s_q, h_q, 128], LSE FP32 [b, h_q, s_q]."""
    import torch
    if o_parts.dtype != torch.float32 or lse_parts.dtype != torch.float32:
        raise TypeError("partials must be float32")
    if o_parts.dim() != 5 or lse_parts.dim() != 4 or not o_parts.is_contiguous() \
            or not lse_parts.is_contiguous():
        raise ValueError("o_parts [n, b, h, s, d] and lse_parts [n, b, h, s], contiguous")
    n, b, h_q, s_q, d = o_parts.shape
    if tuple(lse_parts.shape) != (n, b, h_q, s_q):
        raise ValueError("o_parts and lse_parts shapes disagree")
    dev = _cuda_device(stream, o_parts=o_parts, lse_parts=lse_parts)
    with _on_device(dev):
        o, lse = _outputs(o_parts, o, lse, (b, s_q, h_q, d), (b, h_q, s_q), stream)
        rc = load_library().attn_merge_partials(o_parts.data_ptr(), lse_parts.data_ptr(), n, b,
                                                h_q, s_q, d, o.data_ptr(), lse.data_ptr(),
                                                _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_merge_partials")
    return o, lse


def attn_fwd_raw(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, b, h_q, h_kv, s_q, s_k, d, causal, scale,
                 stream_handle) -> int:
    """Direct call of the C entry point (buffers on the current device);
    returns its status code."""
    return load_library().attn_fwd(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, b, h_q, h_kv, s_q, s_k,
                                   d, int(causal), float(scale), stream_handle)


def host_workspace_bytes(b, h_q, h_kv, s_q, s_k, d=128) -> int:
    return int(load_library().attn_fwd_host_workspace_bytes(b, h_q, h_kv, s_q, s_k, d))


def attn_fwd_host(q, k, v, o, lse, workspace, causal: bool = False, scale: float | None = None,
                  stream=None):
    """Forward on HOST tensors (pinned for asynchronous copies) through the
    C entry point that copies in, runs and copies out.  ``workspace`` is a
    CUDA uint8 tensor of at least :func:`host_workspace_bytes` bytes; the
    call runs on its device."""
    import torch
    b, s_q, h_q, h_kv, s_k, d = _check_qkv(q, k, v)
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.is_cuda:
            raise ValueError(f"{name} must be a host tensor (attn_fwd takes device tensors)")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    _check_out(o, "o", (b, s_q, h_q, d), torch.bfloat16, q.device)
    _check_out(lse, "lse", (b, h_q, s_q), torch.float32, q.device)
    dev = _cuda_device(stream, workspace=workspace)
    if not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    with _on_device(dev):
        rc = load_library().attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                          o.data_ptr(), lse.data_ptr(), b, h_q, h_kv, s_q, s_k,
                                          d, int(bool(causal)), float(scale),
                                          workspace.data_ptr(), _nbytes(workspace),
                                          _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_host")
    return o, lse


def attn_status(stream=None) -> int:
    """Synchronise the stream, then read and clear the status word of the
    current device (the status word is per device: call this with the device
    of the launches it should cover current, e.g. under
    ``torch.cuda.device(q.device)``)."""
    return int(load_library().attn_status(_stream_handle(stream)))


def set_wait_timeout_ns(ns: int) -> None:
    """Bound on every device-side wait of kernels launched afterwards (0: the
    default, 2 s)."""
    if int(ns) < 0:
        raise ValueError("the timeout is a non-negative number of nanoseconds")
    rc = load_library().attn_set_wait_timeout_ns(int(ns))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_set_wait_timeout_ns")


def selftest_wait_timeout(timeout_ns: int, stream=None) -> int:
    return int(load_library().attn_selftest_wait_timeout(int(timeout_ns), _stream_handle(stream)))


def last_launch_count() -> int:
    return int(load_library().attn_last_launch_count())

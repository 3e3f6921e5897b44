"""Python binding of libgqa: one grouped-query-attention decode step on B200.

This module only marshals arguments: it takes torch tensors (device memory the caller
allocated), passes their pointers, sizes and the current CUDA stream to the C ABI declared in
``include/gqa.h``, and turns error codes into exceptions.  Every step of the computation runs in
the library's CUDA kernels; there is no fallback.  If ``libgqa.so`` has not been built, importing
the binding's functions raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgqa.so")

DTYPE_F32 = 0
DTYPE_BF16 = 1
_DTYPES = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}

# status bits written by the kernels (include/gqa.h)
STATUS_APPEND_OVERFLOW = 1
STATUS_SEQLEN_RANGE = 2
STATUS_WAIT_TIMEOUT = 4
STATUS_INTERNAL = 8
STATUS_PAGE_RANGE = 16

# C-ABI symbols declared in include/gqa.h
EXPORTED = ("gqa_kv_append", "gqa_decode_workspace_size", "gqa_decode", "gqa_status_string",
            "gqa_set_wait_timeout_ns", "gqa_profile_events", "gqa_decode_noalloc",
            "gqa_decode_window", "gqa_kv_append_paged", "gqa_decode_paged",
            "gqa_kv_append_multi", "gqa_decode_multi_workspace_size", "gqa_decode_multi",
            "gqa_kv_append_fp8", "gqa_kv_append_paged_fp8", "gqa_decode_fp8",
            "gqa_decode_paged_fp8", "gqa_kv_append_decode")


class GQAError(RuntimeError):
    """A libgqa call returned a negative GQA_ERR_* code."""

    def __init__(self, code: int, msg: str):
        super().__init__(f"libgqa error {code}: {msg}")
        self.code = code


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libgqa.so (once).  Raises OSError when it is missing: build it first with
    ``python -m grouped_query_attention_decode_b200.build``."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"{path} not found; build it with `python -m grouped_query_attention_decode_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32p = ctypes.c_void_p, ctypes.c_void_p
    c_int, c_size = ctypes.c_int, ctypes.c_size_t
    lib.gqa_kv_append.argtypes = [vp, vp, vp, vp, i32p, c_int, c_int, c_int, c_int, c_int, i32p, vp]
    lib.gqa_kv_append.restype = c_int
    lib.gqa_decode_workspace_size.argtypes = [c_int, c_int, c_int, c_int, c_int]
    lib.gqa_decode_workspace_size.restype = c_size
    lib.gqa_decode.argtypes = [vp, vp, vp, i32p, c_int, c_int, c_int, c_int, c_int,
                               ctypes.c_float, c_int, vp, vp, c_size, i32p, vp]
    lib.gqa_decode.restype = c_int
    lib.gqa_kv_append_decode.argtypes = [vp, vp, vp, vp, vp, i32p, i32p, c_int, c_int, c_int,
                                         c_int, c_int, ctypes.c_float, c_int, vp, vp, c_size,
                                         i32p, vp]
    lib.gqa_kv_append_decode.restype = c_int
    lib.gqa_decode_window.argtypes = [vp, vp, vp, i32p, c_int, c_int, c_int, c_int, c_int, c_int,
                                      ctypes.c_float, c_int, vp, vp, c_size, i32p, vp]
    lib.gqa_decode_window.restype = c_int
    lib.gqa_kv_append_paged.argtypes = [vp, vp, vp, vp, i32p, c_int, i32p, c_int, c_int, c_int,
                                        c_int, c_int, c_int, i32p, vp]
    lib.gqa_kv_append_paged.restype = c_int
    lib.gqa_decode_paged.argtypes = [vp, vp, vp, i32p, c_int, i32p, c_int, c_int, c_int, c_int,
                                     c_int, c_int, ctypes.c_float, c_int, vp, vp, c_size, i32p, vp]
    lib.gqa_decode_paged.restype = c_int
    lib.gqa_kv_append_multi.argtypes = [vp, vp, vp, vp, i32p, c_int, c_int, c_int, c_int, c_int,
                                        c_int, i32p, vp]
    lib.gqa_kv_append_multi.restype = c_int
    lib.gqa_decode_multi_workspace_size.argtypes = [c_int, c_int, c_int, c_int, c_int, c_int]
    lib.gqa_decode_multi_workspace_size.restype = c_size
    lib.gqa_decode_multi.argtypes = [vp, vp, vp, i32p, c_int, c_int, c_int, c_int, c_int, c_int,
                                     ctypes.c_float, c_int, vp, vp, c_size, i32p, vp]
    lib.gqa_decode_multi.restype = c_int
    lib.gqa_decode_noalloc.argtypes = [vp, vp, vp, i32p, c_int, c_int, c_int, c_int, c_int,
                                       ctypes.c_float, c_int, vp, i32p, vp]
    lib.gqa_decode_noalloc.restype = c_int
    fp = ctypes.POINTER(ctypes.c_float)
    lib.gqa_kv_append_fp8.argtypes = [vp, vp, c_int, vp, vp, vp, vp, i32p, c_int, c_int, c_int,
                                      c_int, i32p, vp]
    lib.gqa_kv_append_fp8.restype = c_int
    lib.gqa_kv_append_paged_fp8.argtypes = [vp, vp, c_int, vp, vp, vp, vp, i32p, c_int, i32p,
                                            c_int, c_int, c_int, c_int, c_int, i32p, vp]
    lib.gqa_kv_append_paged_fp8.restype = c_int
    lib.gqa_decode_fp8.argtypes = [vp, vp, vp, vp, vp, i32p, c_int, c_int, c_int, c_int, c_int,
                                   c_int, ctypes.c_float, vp, vp, ctypes.c_size_t, i32p, vp]
    lib.gqa_decode_fp8.restype = c_int
    lib.gqa_decode_paged_fp8.argtypes = [vp, vp, vp, vp, vp, i32p, c_int, i32p, c_int, c_int,
                                         c_int, c_int, c_int, c_int, ctypes.c_float, vp, vp,
                                         ctypes.c_size_t, i32p, vp]
    lib.gqa_decode_paged_fp8.restype = c_int
    lib.gqa_status_string.argtypes = [c_int]
    lib.gqa_status_string.restype = ctypes.c_char_p
    lib.gqa_set_wait_timeout_ns.argtypes = [ctypes.c_ulonglong]
    lib.gqa_set_wait_timeout_ns.restype = c_int
    lib.gqa_profile_events.argtypes = [vp, vp]
    lib.gqa_profile_events.restype = c_int
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load_library().gqa_status_string(int(code)).decode()


def _check(rc: int):
    if rc != 0:
        raise GQAError(rc, status_string(rc))


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("libgqa needs contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {t.dtype}")
    return _DTYPES[t.dtype]


def kv_append(k_new, v_new, k_cache, v_cache, seq_lens, status=None, stream=None) -> None:
    """gqa_kv_append: k_cache[b, seq_lens[b]] = k_new[b] (and V), then seq_lens[b] += 1."""
    B, L_max, H_kv, d = k_cache.shape
    _check(load_library().gqa_kv_append(
        _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens),
        B, H_kv, d, L_max, _dtype(k_cache), _ptr(status), _stream(stream)))


def workspace_size(B: int, H_q: int, H_kv: int, d: int, dtype: torch.dtype) -> int:
    """Bytes of workspace gqa_decode needs on the current device."""
    return int(load_library().gqa_decode_workspace_size(B, H_q, H_kv, d, _DTYPES[dtype]))


def alloc_workspace(B: int, H_q: int, H_kv: int, d: int, dtype: torch.dtype, device=None):
    n = workspace_size(B, H_q, H_kv, d, dtype)
    if n == 0:
        raise GQAError(-9, "no usable sm_100 device is current, or invalid sizes")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def decode(q, k_cache, v_cache, seq_lens, scale: float, out=None, workspace=None, status=None,
           stream=None) -> torch.Tensor:
    """gqa_decode: attention of one decode step.  Returns ``out`` [B, H_q, d] float32."""
    B, H_q, d = q.shape
    _, L_max, H_kv, _ = k_cache.shape
    if out is None:
        out = torch.empty((B, H_q, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(B, H_q, H_kv, d, k_cache.dtype, device=q.device)
    _check(load_library().gqa_decode(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), B, H_q, H_kv, d, L_max,
        float(scale), _dtype(k_cache), _ptr(out), _ptr(workspace), workspace.numel(),
        _ptr(status), _stream(stream)))
    return out


def kv_append_decode(q, k_new, v_new, k_cache, v_cache, seq_lens, seq_lens_out, scale: float,
                     out=None, workspace=None, status=None, stream=None) -> torch.Tensor:
    """gqa_kv_append_decode: append k_new/v_new at row seq_lens[b] and attend the rows up to and
    including it, in one launch; the new lengths go to ``seq_lens_out`` (``seq_lens`` is only
    read).  Returns ``out`` [B, H_q, d] float32."""
    B, H_q, d = q.shape
    _, L_max, H_kv, _ = k_cache.shape
    if out is None:
        out = torch.empty((B, H_q, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(B, H_q, H_kv, d, k_cache.dtype, device=q.device)
    _check(load_library().gqa_kv_append_decode(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens),
        _ptr(seq_lens_out), B, H_q, H_kv, d, L_max, float(scale), _dtype(k_cache), _ptr(out),
        _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)))
    return out


def decode_window(q, k_cache, v_cache, seq_lens, window: int, scale: float, out=None,
                  workspace=None, status=None, stream=None) -> torch.Tensor:
    """gqa_decode_window: each sequence attends only its last ``window`` cached rows."""
    B, H_q, d = q.shape
    _, L_max, H_kv, _ = k_cache.shape
    if out is None:
        out = torch.empty((B, H_q, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(B, H_q, H_kv, d, k_cache.dtype, device=q.device)
    _check(load_library().gqa_decode_window(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), B, H_q, H_kv, d, L_max,
        int(window), float(scale), _dtype(k_cache), _ptr(out), _ptr(workspace),
        workspace.numel(), _ptr(status), _stream(stream)))
    return out


def kv_append_paged(k_new, v_new, k_pool, v_pool, block_table, seq_lens, status=None,
                    stream=None) -> None:
    """gqa_kv_append_paged: pools [n_pages, page_size, H_kv, d], block_table [B, max_pages]."""
    n_pages, page_size, H_kv, d = k_pool.shape
    B, max_pages = block_table.shape
    _check(load_library().gqa_kv_append_paged(
        _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool), _ptr(block_table), max_pages,
        _ptr(seq_lens), B, H_kv, d, page_size, n_pages, _dtype(k_pool), _ptr(status),
        _stream(stream)))


def decode_paged(q, k_pool, v_pool, block_table, seq_lens, scale: float, out=None,
                 workspace=None, status=None, stream=None) -> torch.Tensor:
    """gqa_decode_paged: the decode over a paged cache."""
    B, H_q, d = q.shape
    n_pages, page_size, H_kv, _ = k_pool.shape
    _, max_pages = block_table.shape
    if out is None:
        out = torch.empty((B, H_q, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(B, H_q, H_kv, d, k_pool.dtype, device=q.device)
    _check(load_library().gqa_decode_paged(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_table), max_pages, _ptr(seq_lens), B,
        H_q, H_kv, d, page_size, n_pages, float(scale), _dtype(k_pool), _ptr(out),
        _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)))
    return out


def kv_append_multi(k_new, v_new, k_cache, v_cache, seq_lens, status=None, stream=None) -> None:
    """gqa_kv_append_multi: k_new, v_new [B, Q, H_kv, d] to rows seq_lens[b] .. + Q - 1."""
    B, L_max, H_kv, d = k_cache.shape
    Q = k_new.shape[1]
    _check(load_library().gqa_kv_append_multi(
        _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), B, Q, H_kv, d,
        L_max, _dtype(k_cache), _ptr(status), _stream(stream)))


def decode_multi(q, k_cache, v_cache, seq_lens, scale: float, out=None, workspace=None,
                 status=None, stream=None) -> torch.Tensor:
    """gqa_decode_multi: q [B, Q, H_q, d]; token j attends rows [0, n - Q + 1 + j)."""
    B, Q, H_q, d = q.shape
    _, L_max, H_kv, _ = k_cache.shape
    lib = load_library()
    if out is None:
        out = torch.empty((B, Q, H_q, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        n = int(lib.gqa_decode_multi_workspace_size(B, Q, H_q, H_kv, d, _DTYPES[k_cache.dtype]))
        if n == 0:
            raise GQAError(-9, "no usable sm_100 device is current, or invalid sizes")
        workspace = torch.zeros(n, dtype=torch.uint8, device=q.device)
    _check(lib.gqa_decode_multi(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), B, Q, H_q, H_kv, d, L_max,
        float(scale), _dtype(k_cache), _ptr(out), _ptr(workspace), workspace.numel(),
        _ptr(status), _stream(stream)))
    return out


def decode_noalloc(q, k_cache, v_cache, seq_lens, scale: float, out=None, status=None,
                   stream=None) -> torch.Tensor:
    """gqa_decode_noalloc: like ``decode`` but with the library's own fixed scratch array
    instead of a caller workspace (for callers that cannot allocate one).  Calls that may run
    at the same time on the GPU must not overlap: they share that array."""
    B, H_q, d = q.shape
    _, L_max, H_kv, _ = k_cache.shape
    if out is None:
        out = torch.empty((B, H_q, d), dtype=torch.float32, device=q.device)
    _check(load_library().gqa_decode_noalloc(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), B, H_q, H_kv, d, L_max,
        float(scale), _dtype(k_cache), _ptr(out), _ptr(status), _stream(stream)))
    return out


def set_wait_timeout_ns(ns: int) -> None:
    """Time limit of the decode kernels' internal waits (0 restores the 2 s default)."""
    _check(load_library().gqa_set_wait_timeout_ns(int(ns)))


def profile_events(before_split=None, after_split=None) -> None:
    """Record these torch.cuda.Events around every later split-KV kernel (None, None stops)."""
    a = ctypes.c_void_p(before_split.cuda_event) if before_split is not None else None
    b = ctypes.c_void_p(after_split.cuda_event) if after_split is not None else None
    _check(load_library().gqa_profile_events(a, b))


# ------------------------------------------------------------------ FP8 (e4m3) cache
DTYPE_E4M3 = 2


def _codes(t: torch.Tensor) -> torch.Tensor:
    """An e4m3 cache as bytes: torch.uint8, or torch.float8_e4m3fn viewed as uint8."""
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8)
    if t.dtype != torch.uint8:
        raise ValueError(f"an e4m3 cache must be uint8 or float8_e4m3fn, not {t.dtype}")
    return t


def _scales(t: torch.Tensor, H_kv: int) -> torch.Tensor:
    if t.dtype != torch.float32 or t.shape != (H_kv,):
        raise ValueError(f"scales must be float32 [{H_kv}]")
    return t


def alloc_workspace_fp8(B: int, H_q: int, H_kv: int, d: int, device=None):
    n = int(load_library().gqa_decode_workspace_size(B, H_q, H_kv, d, DTYPE_E4M3))
    if n == 0:
        raise GQAError(-9, "no usable sm_100 device is current, or invalid sizes")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def kv_append_fp8(k_new, v_new, k_cache, v_cache, k_scale, v_scale, seq_lens, status=None,
                  stream=None) -> None:
    """gqa_kv_append_fp8: quantise k_new/v_new [B, H_kv, d] (bf16 or float32) to e4m3 codes of
    their head's scale and write them at row seq_lens[b]; then seq_lens[b] += 1."""
    kc, vc = _codes(k_cache), _codes(v_cache)
    B, L_max, H_kv, d = kc.shape
    _check(load_library().gqa_kv_append_fp8(
        _ptr(k_new), _ptr(v_new), _dtype(k_new), _ptr(kc), _ptr(vc),
        _ptr(_scales(k_scale, H_kv)), _ptr(_scales(v_scale, H_kv)), _ptr(seq_lens), B, H_kv, d,
        L_max, _ptr(status), _stream(stream)))


def kv_append_paged_fp8(k_new, v_new, k_pool, v_pool, k_scale, v_scale, block_table, seq_lens,
                        status=None, stream=None) -> None:
    """gqa_kv_append_paged_fp8: the quantising append into e4m3 page pools."""
    kp, vp_ = _codes(k_pool), _codes(v_pool)
    n_pages, page_size, H_kv, d = kp.shape
    B, max_pages = block_table.shape
    _check(load_library().gqa_kv_append_paged_fp8(
        _ptr(k_new), _ptr(v_new), _dtype(k_new), _ptr(kp), _ptr(vp_),
        _ptr(_scales(k_scale, H_kv)), _ptr(_scales(v_scale, H_kv)), _ptr(block_table), max_pages,
        _ptr(seq_lens), B, H_kv, d, page_size, n_pages, _ptr(status), _stream(stream)))


def decode_fp8(q, k_cache, v_cache, k_scale, v_scale, seq_lens, scale: float, window: int = 0,
               out=None, workspace=None, status=None, stream=None) -> torch.Tensor:
    """gqa_decode_fp8: the decode over an e4m3 cache (window > 0: sliding window).  q is bf16
    [B, H_q, d]; returns out [B, H_q, d] float32."""
    kc, vc = _codes(k_cache), _codes(v_cache)
    B, H_q, d = q.shape
    _, L_max, H_kv, _ = kc.shape
    if q.dtype != torch.bfloat16:
        raise ValueError("q must be bfloat16 for an e4m3 cache")
    if out is None:
        out = torch.empty((B, H_q, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace_fp8(B, H_q, H_kv, d, device=q.device)
    _check(load_library().gqa_decode_fp8(
        _ptr(q), _ptr(kc), _ptr(vc), _ptr(_scales(k_scale, H_kv)), _ptr(_scales(v_scale, H_kv)),
        _ptr(seq_lens), B, H_q, H_kv, d, L_max, int(window), float(scale), _ptr(out),
        _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)))
    return out


def decode_paged_fp8(q, k_pool, v_pool, k_scale, v_scale, block_table, seq_lens, scale: float,
                     out=None, workspace=None, status=None, stream=None) -> torch.Tensor:
    """gqa_decode_paged_fp8: the decode over e4m3 page pools."""
    kp, vp_ = _codes(k_pool), _codes(v_pool)
    B, H_q, d = q.shape
    n_pages, page_size, H_kv, _ = kp.shape
    _, max_pages = block_table.shape
    if q.dtype != torch.bfloat16:
        raise ValueError("q must be bfloat16 for an e4m3 cache")
    if out is None:
        out = torch.empty((B, H_q, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace_fp8(B, H_q, H_kv, d, device=q.device)
    _check(load_library().gqa_decode_paged_fp8(
        _ptr(q), _ptr(kp), _ptr(vp_), _ptr(_scales(k_scale, H_kv)), _ptr(_scales(v_scale, H_kv)),
        _ptr(block_table), max_pages, _ptr(seq_lens), B, H_q, H_kv, d, page_size, n_pages,
        float(scale), _ptr(out), _ptr(workspace), workspace.numel(), _ptr(status),
        _stream(stream)))
    return out

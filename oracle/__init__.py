"""CPU float64 oracle for one grouped-query-attention decode step.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg are the only callers.  The CUDA library never imports, links or runs anything
here, and nothing here imports the CUDA library.

The arithmetic lives in ``gqa_oracle.c`` (plain C, float64); this module compiles it with gcc
and marshals numpy arrays to it.  ``counts.py`` holds the cache-size and multiply-count
formulas of the pages.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gqa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

APPEND_OVERFLOW = 1
SEQLEN_RANGE = 2
PAGE_RANGE = 4  # a block-table entry outside the pool for a row below the length


def build(src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (OpenMP over query heads, no fast-math)."""
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _needs_build(src: str, lib: str) -> bool:
    return not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src)


class Oracle:
    """ctypes view of one compiled oracle library (the default one, or a test's variant)."""

    def __init__(self, lib_path: str | None = None):
        if lib_path is None:
            if _needs_build(_SRC, _LIB):
                build()
            lib_path = _LIB
        self.lib = ctypes.CDLL(lib_path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        c_int = ctypes.c_int
        self.lib.oracle_kv_append.argtypes = [dp, dp, dp, dp, ip, c_int, c_int, c_int, c_int, ip]
        self.lib.oracle_kv_append.restype = None
        self.lib.oracle_expand_kv.argtypes = [dp, c_int, c_int, c_int, c_int, dp]
        self.lib.oracle_expand_kv.restype = None
        self.lib.oracle_attend_one_head.argtypes = [dp, dp, dp, c_int, c_int, ctypes.c_size_t,
                                                    ctypes.c_double, dp, dp]
        self.lib.oracle_attend_one_head.restype = None
        self.lib.oracle_gqa_decode.argtypes = [dp, dp, dp, ip, c_int, c_int, c_int, c_int, c_int,
                                               ctypes.c_double, dp, c_int, ip]
        self.lib.oracle_gqa_decode.restype = c_int
        self.lib.oracle_gqa_decode_window.argtypes = [dp, dp, dp, ip, c_int, c_int, c_int, c_int,
                                                      c_int, c_int, ctypes.c_double, dp, c_int, ip]
        self.lib.oracle_gqa_decode_window.restype = c_int
        self.lib.oracle_paged_gather.argtypes = [dp, ip, ip, c_int, c_int, c_int, c_int, c_int,
                                                 c_int, dp, ip]
        self.lib.oracle_paged_gather.restype = None
        self.lib.oracle_kv_append_paged.argtypes = [dp, dp, dp, dp, ip, ip, c_int, c_int, c_int,
                                                    c_int, c_int, c_int, ip]
        self.lib.oracle_kv_append_paged.restype = None
        self.lib.oracle_gqa_decode_multi.argtypes = [dp, dp, dp, ip, c_int, c_int, c_int, c_int,
                                                     c_int, c_int, ctypes.c_double, dp, c_int, ip]
        self.lib.oracle_gqa_decode_multi.restype = c_int
        u8p = ctypes.POINTER(ctypes.c_uint8)
        fp = ctypes.POINTER(ctypes.c_float)
        self.lib.oracle_e4m3_value.argtypes = [c_int]
        self.lib.oracle_e4m3_value.restype = ctypes.c_double
        self.lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        self.lib.oracle_e4m3_encode.restype = c_int
        self.lib.oracle_e4m3_values.argtypes = [u8p, ctypes.c_size_t, dp]
        self.lib.oracle_e4m3_values.restype = None
        self.lib.oracle_e4m3_encode_array.argtypes = [fp, ctypes.c_size_t, u8p]
        self.lib.oracle_e4m3_encode_array.restype = None
        self.lib.oracle_quantize_rows.argtypes = [dp, ctypes.c_size_t, c_int, c_int, fp, u8p]
        self.lib.oracle_quantize_rows.restype = None
        self.lib.oracle_dequantize_rows.argtypes = [u8p, ctypes.c_size_t, c_int, c_int, fp, dp]
        self.lib.oracle_dequantize_rows.restype = None
        self.lib.oracle_max_threads.argtypes = []
        self.lib.oracle_max_threads.restype = c_int

    @staticmethod
    def _f64(a) -> np.ndarray:
        return np.ascontiguousarray(a, dtype=np.float64)

    @staticmethod
    def _dp(a: np.ndarray):
        return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))

    @staticmethod
    def _ip(a: np.ndarray):
        return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    def kv_append(self, k_new, v_new, k_cache, v_cache, seq_lens):
        """Append one K/V row per (sequence, kv-head).  k_cache/v_cache ([B, L_max, H_kv, d]
        float64) and seq_lens ([B] int32) are updated in place.  Returns the status bits."""
        assert k_cache.dtype == np.float64 and k_cache.flags.c_contiguous
        assert v_cache.dtype == np.float64 and v_cache.flags.c_contiguous
        assert seq_lens.dtype == np.int32 and seq_lens.flags.c_contiguous
        B, L_max, H_kv, d = k_cache.shape
        kn, vn = self._f64(k_new), self._f64(v_new)
        status = np.zeros(1, dtype=np.int32)
        self.lib.oracle_kv_append(self._dp(kn), self._dp(vn), self._dp(k_cache), self._dp(v_cache),
                                  self._ip(seq_lens), B, H_kv, d, L_max, self._ip(status))
        return int(status[0])

    def expand_kv(self, cache_b, n: int, H_q: int):
        """Repeat the key/value heads of one sequence ([L_max, H_kv, d]) to [n, H_q, d]."""
        c = self._f64(cache_b)
        _, H_kv, d = c.shape
        out = np.empty((n, H_q, d), dtype=np.float64)
        self.lib.oracle_expand_kv(self._dp(c), n, H_q, H_kv, d, self._dp(out))
        return out

    def attend_one_head(self, q, K, V, scale: float):
        """Single-head softmax attention of q [d] over rows K, V [n, d].  Returns (out, weights)."""
        q, K, V = self._f64(q), self._f64(K), self._f64(V)
        n, d = K.shape
        out = np.empty(d, dtype=np.float64)
        w = np.empty(max(n, 1), dtype=np.float64)
        self.lib.oracle_attend_one_head(self._dp(q), self._dp(K), self._dp(V), n, d, d, scale,
                                        self._dp(out), self._dp(w))
        return out, w[:n]

    def decode(self, q, k_cache, v_cache, seq_lens, scale: float, nthreads: int = 0,
               return_status: bool = False):
        """out[b, h, :] = softmax(scale * q[b,h] . K[b, :n_b, h // r]^T) . V[b, :n_b, h // r]."""
        q, kc, vc = self._f64(q), self._f64(k_cache), self._f64(v_cache)
        lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
        B, H_q, d = q.shape
        Bk, L_max, H_kv, dk = kc.shape
        assert Bk == B and dk == d and vc.shape == kc.shape and lens.shape == (B,)
        out = np.zeros((B, H_q, d), dtype=np.float64)
        status = np.zeros(1, dtype=np.int32)
        rc = self.lib.oracle_gqa_decode(self._dp(q), self._dp(kc), self._dp(vc), self._ip(lens),
                                        B, H_q, H_kv, d, L_max, float(scale), self._dp(out),
                                        int(nthreads), self._ip(status))
        if rc != 0:
            raise ValueError("oracle_gqa_decode rejected the shapes (H_q % H_kv != 0?)")
        return (out, int(status[0])) if return_status else out


    def decode_window(self, q, k_cache, v_cache, seq_lens, window: int, scale: float,
                      nthreads: int = 0):
        """Like decode, but each sequence attends only its last `window` rows (window <= 0:
        all rows)."""
        q, kc, vc = self._f64(q), self._f64(k_cache), self._f64(v_cache)
        lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
        B, H_q, d = q.shape
        _, L_max, H_kv, _ = kc.shape
        out = np.zeros((B, H_q, d), dtype=np.float64)
        status = np.zeros(1, dtype=np.int32)
        rc = self.lib.oracle_gqa_decode_window(self._dp(q), self._dp(kc), self._dp(vc),
                                               self._ip(lens), B, H_q, H_kv, d, L_max, int(window),
                                               float(scale), self._dp(out), int(nthreads),
                                               self._ip(status))
        if rc != 0:
            raise ValueError("oracle_gqa_decode_window rejected the shapes")
        return out


    def decode_multi(self, q, k_cache, v_cache, seq_lens, scale: float, nthreads: int = 0,
                     return_status: bool = False):
        """Q query tokens per sequence (q [B, Q, H_q, d]); query j attends rows
        [0, n - Q + 1 + j).  Returns out [B, Q, H_q, d]."""
        q, kc, vc = self._f64(q), self._f64(k_cache), self._f64(v_cache)
        lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
        B, Q, H_q, d = q.shape
        _, L_max, H_kv, _ = kc.shape
        out = np.zeros((B, Q, H_q, d), dtype=np.float64)
        status = np.zeros(1, dtype=np.int32)
        rc = self.lib.oracle_gqa_decode_multi(self._dp(q), self._dp(kc), self._dp(vc), self._ip(lens),
                                              B, Q, H_q, H_kv, d, L_max, float(scale), self._dp(out),
                                              int(nthreads), self._ip(status))
        if rc != 0:
            raise ValueError("oracle_gqa_decode_multi rejected the shapes")
        return (out, int(status[0])) if return_status else out

    def paged_gather(self, pool, block_table, seq_lens):
        """Logical caches [B, max_pages*page_size, H_kv, d] of a paged pool
        [n_pages, page_size, H_kv, d]; rows >= seq_lens[b] are zero.  Returns (cache, status)."""
        pool = self._f64(pool)
        bt = np.ascontiguousarray(block_table, dtype=np.int32)
        lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
        n_pages, P, H_kv, d = pool.shape
        B, max_pages = bt.shape
        cache = np.zeros((B, max_pages * P, H_kv, d), dtype=np.float64)
        status = np.zeros(1, dtype=np.int32)
        self.lib.oracle_paged_gather(self._dp(pool), self._ip(bt), self._ip(lens), B, max_pages, P,
                                     n_pages, H_kv, d, self._dp(cache), self._ip(status))
        return cache, int(status[0])

    def kv_append_paged(self, k_new, v_new, k_pool, v_pool, block_table, seq_lens):
        """Paged append (in place on the float64 pools and int32 lengths).  Returns status."""
        assert k_pool.dtype == np.float64 and k_pool.flags.c_contiguous
        assert v_pool.dtype == np.float64 and v_pool.flags.c_contiguous
        assert seq_lens.dtype == np.int32 and seq_lens.flags.c_contiguous
        bt = np.ascontiguousarray(block_table, dtype=np.int32)
        n_pages, P, H_kv, d = k_pool.shape
        B, max_pages = bt.shape
        kn, vn = self._f64(k_new), self._f64(v_new)
        status = np.zeros(1, dtype=np.int32)
        self.lib.oracle_kv_append_paged(self._dp(kn), self._dp(vn), self._dp(k_pool), self._dp(v_pool),
                                        self._ip(bt), self._ip(seq_lens), B, max_pages, P, n_pages,
                                        H_kv, d, self._ip(status))
        return int(status[0])

    def decode_paged(self, q, k_pool, v_pool, block_table, seq_lens, scale: float,
                     return_status: bool = False):
        """The paged decode: gather each sequence's rows from the pool, then decode.  With
        return_status, also returns the status bits of the gathers and the decode (PAGE_RANGE
        when a block-table entry for a row below the length lies outside the pool; that row is
        then gathered as zeros)."""
        kc, st1 = self.paged_gather(k_pool, block_table, seq_lens)
        vc, st2 = self.paged_gather(v_pool, block_table, seq_lens)
        out, st3 = self.decode(q, kc, vc, seq_lens, scale, return_status=True)
        return (out, st1 | st2 | st3) if return_status else out

    # ------------------------------------------------------------------ FP8 (e4m3) cache
    @staticmethod
    def _u8(a) -> np.ndarray:
        return np.ascontiguousarray(a, dtype=np.uint8)

    @staticmethod
    def _f32(a) -> np.ndarray:
        return np.ascontiguousarray(a, dtype=np.float32)

    def e4m3_values(self, codes):
        """float64 value of every e4m3 code (NaN for 0x7F / 0xFF)."""
        c = self._u8(codes)
        out = np.empty(c.shape, dtype=np.float64)
        self.lib.oracle_e4m3_values(c.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), c.size,
                                    self._dp(out))
        return out

    def e4m3_encode(self, x):
        """Nearest finite e4m3 code of every float32 in x (ties to even, saturating)."""
        xf = self._f32(x)
        out = np.empty(xf.shape, dtype=np.uint8)
        self.lib.oracle_e4m3_encode_array(xf.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                                          xf.size, out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
        return out

    def quantize(self, x, scale):
        """Codes of x [..., H_kv, d] (float32 values) with per-head scales [H_kv]."""
        xd = self._f64(x)
        sc = self._f32(scale)
        H_kv, d = xd.shape[-2:]
        assert sc.shape == (H_kv,)
        out = np.empty(xd.shape, dtype=np.uint8)
        self.lib.oracle_quantize_rows(self._dp(xd), xd.size // (H_kv * d), H_kv, d,
                                      sc.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                                      out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
        return out

    def dequantize(self, codes, scale):
        """float64 values value(code) * scale[g] of codes [..., H_kv, d]."""
        c = self._u8(codes)
        sc = self._f32(scale)
        H_kv, d = c.shape[-2:]
        assert sc.shape == (H_kv,)
        out = np.empty(c.shape, dtype=np.float64)
        self.lib.oracle_dequantize_rows(c.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                                        c.size // (H_kv * d), H_kv, d,
                                        sc.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), self._dp(out))
        return out

    def kv_append_fp8(self, k_new, v_new, k_codes, v_codes, k_scale, v_scale, seq_lens):
        """Quantise the new rows and append them to uint8 code caches [B, L_max, H_kv, d]
        (in place, with seq_lens).  Returns the status bits."""
        assert k_codes.dtype == np.uint8 and v_codes.dtype == np.uint8
        kq = self.quantize(k_new, k_scale).astype(np.float64)
        vq = self.quantize(v_new, v_scale).astype(np.float64)
        kc = k_codes.astype(np.float64)
        vc = v_codes.astype(np.float64)
        st = self.kv_append(kq, vq, kc, vc, seq_lens)
        k_codes[...] = kc.astype(np.uint8)
        v_codes[...] = vc.astype(np.uint8)
        return st

    def kv_append_paged_fp8(self, k_new, v_new, k_pool, v_pool, k_scale, v_scale, block_table,
                            seq_lens):
        """Paged form of kv_append_fp8 on uint8 code pools [n_pages, page_size, H_kv, d]."""
        assert k_pool.dtype == np.uint8 and v_pool.dtype == np.uint8
        kq = self.quantize(k_new, k_scale).astype(np.float64)
        vq = self.quantize(v_new, v_scale).astype(np.float64)
        kp = k_pool.astype(np.float64)
        vp = v_pool.astype(np.float64)
        st = self.kv_append_paged(kq, vq, kp, vp, block_table, seq_lens)
        k_pool[...] = kp.astype(np.uint8)
        v_pool[...] = vp.astype(np.uint8)
        return st

    def decode_fp8(self, q, k_codes, v_codes, k_scale, v_scale, seq_lens, scale: float,
                   window: int = 0, nthreads: int = 0):
        """Decode over an e4m3 cache: the oracle decode on the dequantised values."""
        kc = self.dequantize(k_codes, k_scale)
        vc = self.dequantize(v_codes, v_scale)
        return self.decode_window(q, kc, vc, seq_lens, window, scale, nthreads=nthreads)

    def decode_paged_fp8(self, q, k_pool, v_pool, k_scale, v_scale, block_table, seq_lens,
                         scale: float, return_status: bool = False):
        """Paged decode over e4m3 pools: dequantise the pools, gather, decode."""
        return self.decode_paged(q, self.dequantize(k_pool, k_scale),
                                 self.dequantize(v_pool, v_scale), block_table, seq_lens, scale,
                                 return_status=return_status)


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle compiled from ``gqa_oracle.c`` (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default

"""The C-ABI library on the CPU: it loads, exports every symbol include/gqa.h declares, and its
host-side argument checks return the documented codes before touching a GPU."""
import ctypes
import os
import re

import pytest

import grouped_query_attention_decode_b200 as gqa
from grouped_query_attention_decode_b200 import build as cuda_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa.h")


@pytest.fixture(scope="module")
def lib():
    if cuda_build.needs_build():
        cuda_build.build()
    return gqa.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gqa_\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(gqa.EXPORTED)


def test_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(-11, 1):
        s = gqa.status_string(code)
        assert s and s != "unknown status code", code
    assert gqa.status_string(5) == "unknown status code"


P = ctypes.c_void_p
A16 = P(0x10000)        # aligned fake pointers: never dereferenced by the host checks
A256 = P(0x20000)
MIS = P(0x10008)        # 8-byte aligned only


def _decode(lib, q=A16, kc=A16, vc=A16, lens=A16, B=2, H_q=8, H_kv=2, d=64, L=16, scale=0.125,
            dtype=1, out=A16, ws=A256, ws_bytes=1 << 20, status=None):
    return lib.gqa_decode(q, kc, vc, lens, B, H_q, H_kv, d, L, scale, dtype, out, ws, ws_bytes,
                          status, None)


def test_decode_host_checks(lib):
    assert _decode(lib, q=None) == -1
    assert _decode(lib, out=None) == -1
    assert _decode(lib, B=0) == -2
    assert _decode(lib, L=0) == -2
    assert _decode(lib, H_q=6, H_kv=4) == -3
    assert _decode(lib, d=96) == -4
    assert _decode(lib, dtype=7) == -5
    assert _decode(lib, ws=None) == -7
    assert _decode(lib, q=MIS) == -6
    assert _decode(lib, ws=P(0x10010)) == -6
    assert _decode(lib, scale=float("nan")) == -2


def _noalloc(lib, q=A16, kc=A16, vc=A16, lens=A16, B=2, H_q=8, H_kv=2, d=64, L=16, scale=0.125,
             dtype=1, out=A16, status=None):
    return lib.gqa_decode_noalloc(q, kc, vc, lens, B, H_q, H_kv, d, L, scale, dtype, out, status,
                                  None)


def test_noalloc_host_checks_match_decode(lib):
    """The allocation-free entry point returns gqa_decode's codes for the same bad arguments
    (its checks all run before it queues anything on the stream)."""
    assert _noalloc(lib, q=None) == -1
    assert _noalloc(lib, out=None) == -1
    assert _noalloc(lib, B=0) == -2
    assert _noalloc(lib, L=0) == -2
    assert _noalloc(lib, H_q=6, H_kv=4) == -3
    assert _noalloc(lib, d=96) == -4
    assert _noalloc(lib, dtype=7) == -5
    assert _noalloc(lib, dtype=2) == -5   # e4m3 needs gqa_decode_fp8
    assert _noalloc(lib, q=MIS) == -6
    assert _noalloc(lib, status=P(0x10002)) == -6
    assert _noalloc(lib, scale=float("inf")) == -2


def test_append_decode_host_checks(lib):
    def f(q=A16, kn=A16, vn=A16, kc=A16, vc=A16, lens=P(0x30000), lens_out=P(0x40000), B=2, H_q=8,
          H_kv=2, d=64, L=16, scale=0.125, dtype=1, out=A16, ws=A256, ws_bytes=1 << 20):
        return lib.gqa_kv_append_decode(q, kn, vn, kc, vc, lens, lens_out, B, H_q, H_kv, d, L, scale,
                                        dtype, out, ws, ws_bytes, None, None)
    assert f(kn=None) == -1
    assert f(lens_out=None) == -1
    assert f(dtype=0) == -5       # bf16 only
    assert f(vn=MIS) == -6
    assert f(lens_out=P(0x30004)) == -11   # overlaps seq_lens[1]
    assert f(lens_out=P(0x30000)) == -11   # the same array
    assert f(lens_out=P(0x2fffc)) == -11   # overlaps seq_lens[0]
    assert f(B=0) == -2
    assert f(H_q=6, H_kv=4) == -3


def test_append_host_checks(lib):
    f = lib.gqa_kv_append
    assert f(None, A16, A16, A16, A16, 2, 2, 64, 16, 1, None, None) == -1
    assert f(A16, A16, A16, A16, A16, 0, 2, 64, 16, 1, None, None) == -2
    assert f(A16, A16, A16, A16, A16, 2, 2, 80, 16, 1, None, None) == -4
    assert f(A16, A16, A16, A16, A16, 2, 2, 64, 16, 3, None, None) == -5
    assert f(A16, A16, MIS, A16, A16, 2, 2, 64, 16, 1, None, None) == -6


@pytest.mark.skipif(os.environ.get("CUDA_VISIBLE_DEVICES") is None and __import__("torch").cuda.is_available(),
                    reason="only meaningful without a GPU")
def test_valid_arguments_without_a_gpu_report_no_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _decode(lib) == -9
    assert _noalloc(lib) == -9
    assert lib.gqa_decode_workspace_size(2, 8, 2, 64, 1) == 0
    assert lib.gqa_kv_append(A16, A16, A16, A16, A16, 2, 2, 64, 16, 1, None, None) == -9


def test_setters(lib):
    assert lib.gqa_set_wait_timeout_ns(0) == 0
    assert lib.gqa_profile_events(None, None) == 0

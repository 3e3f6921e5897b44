"""gqa_decode_noalloc, the entry point for callers that cannot allocate a workspace.

Such callers (a plugin whose host framework owns all device memory, a serving loop that must
not call cudaMalloc and has no buffer to lend) get the library's own fixed scratch array.  This
file checks, through the C ABI, that the allocation-free call returns what gqa_decode returns
with a caller workspace (bit for bit: the same kernel runs), on two calls in a row (the second reuses the array the first left
behind), and that sizes needing more scratch than the array holds are refused.  It sits last
in collection order so that a failure here leaves every other test already run.
"""
import ctypes

import pytest
import torch

import grouped_query_attention_decode_b200 as gqa
from grouped_query_attention_decode_b200 import inputs

pytestmark = pytest.mark.gpu

CASES = [
    inputs.custom("noalloc_bf16", B=6, H_q=32, H_kv=8, d=128, L_max=700, dtype=torch.bfloat16,
                  q_std=0.5, kv_std=1.0, seed=71),
    inputs.custom("noalloc_f32", B=2, H_q=8, H_kv=2, d=64, L_max=300, dtype=torch.float32, seed=72),
]


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_workspace_entry_point(w):
    lib = gqa.load_library()
    x = inputs.make_inputs(w)
    dev = torch.device("cuda")
    q, kc, vc = x["q"].to(dev), x["k_cache"].to(dev), x["v_cache"].to(dev)
    lens = x["lengths"].to(dev)
    dt = gqa.DTYPE_BF16 if w.dtype == torch.bfloat16 else gqa.DTYPE_F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    args = (w.B, w.H_q, w.H_kv, w.d, w.L_max, ctypes.c_float(x["scale"]), dt)

    ref = torch.empty((w.B, w.H_q, w.d), dtype=torch.float32, device=dev)
    nbytes = lib.gqa_decode_workspace_size(w.B, w.H_q, w.H_kv, w.d, dt)
    assert 0 < nbytes
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    rc = lib.gqa_decode(_p(q), _p(kc), _p(vc), _p(lens), *args, _p(ref), _p(ws), nbytes,
                        _p(status), stream)
    assert rc == 0, gqa.status_string(rc)

    outs = []
    for _ in range(2):
        out = torch.full((w.B, w.H_q, w.d), float("nan"), dtype=torch.float32, device=dev)
        rc = lib.gqa_decode_noalloc(_p(q), _p(kc), _p(vc), _p(lens), *args, _p(out), _p(status),
                                    stream)
        assert rc == 0, gqa.status_string(rc)
        outs.append(out)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # the same kernel on the same inputs with a fixed merge order: identical bits
    for out in outs:
        assert torch.isfinite(out).all()
        assert torch.equal(out, ref)


def test_noalloc_refuses_sizes_beyond_its_array():
    lib = gqa.load_library()
    # 4096 sequences x 64 query heads need far more than the fixed array; refused before any
    # pointer is touched
    B, H_q, H_kv, d = 4096, 64, 8, 128
    need = lib.gqa_decode_workspace_size(B, H_q, H_kv, d, gqa.DTYPE_BF16)
    assert need > (8 << 20)
    fake = ctypes.c_void_p(0x100000)
    rc = lib.gqa_decode_noalloc(fake, fake, fake, fake, B, H_q, H_kv, d, 4096, ctypes.c_float(0.1),
                                gqa.DTYPE_BF16, fake, None, None)
    assert rc == -10
    assert "scratch" in gqa.status_string(rc)

"""GPU parity of the sliding-window decode (gqa_decode_window) against the oracle.

A sequence of n rows attends its last `window` rows, [max(0, n - window), n) ("GQA 阅读笔记",
what came after GQA: Mistral's W).  Windows that start mid-tile, end mid-tile, cover exactly
one tile, one row, or the whole sequence; rows before the window and past n are NaN, so any
read outside the window poisons the output.
"""
import numpy as np
import pytest
import torch

import grouped_query_attention_decode_b200 as gqa
from gpu_helpers import TOL, to_dev
from grouped_query_attention_decode_b200 import inputs

pytestmark = pytest.mark.gpu


def _poison_outside(x, window):
    kc, vc = x["k_cache"].clone(), x["v_cache"].clone()
    for b, n in enumerate(x["lengths"].tolist()):
        first = max(0, n - window)
        kc[b, :first] = float("nan")
        vc[b, :first] = float("nan")
        kc[b, n:] = float("nan")
        vc[b, n:] = float("nan")
    return kc, vc


def _run(oracle, w, lengths, window, bs=None):
    x = inputs.make_inputs(w, lengths=lengths)
    kc, vc = _poison_outside(x, window)
    g = to_dev(x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gqa.decode_window(g["q"], kc.cuda(), vc.cuda(), g["lengths"], window, x["scale"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.isfinite(out).all()
    bs = list(range(w.B)) if bs is None else bs
    for b in bs:
        ref = oracle.decode_window(x["q"][b:b + 1].double().numpy(), x["k_cache"][b:b + 1].double().numpy(),
                                   x["v_cache"][b:b + 1].double().numpy(), x["lengths"][b:b + 1].numpy(),
                                   window, x["scale"])
        err = float(np.max(np.abs(out[b].cpu().double().numpy() - ref[0])))
        assert err <= TOL[w.dtype], (b, err)
    return out


@pytest.mark.parametrize("window", [1, 7, 128, 129, 300, 5000])
def test_window_bf16(oracle, window):
    w = inputs.custom("win", B=5, H_q=32, H_kv=8, d=128, L_max=5000, dtype=torch.bfloat16, seed=41)
    _run(oracle, w, [1, 130, 257, 4999, 5000], window)


@pytest.mark.parametrize("shape", [(2, 64, 1, 64), (3, 16, 16, 64), (2, 8, 2, 128)],
                         ids=lambda s: "B%d_Hq%d_Hkv%d_d%d" % s)
def test_window_group_sizes(oracle, shape):
    B, H_q, H_kv, d = shape
    w = inputs.custom("winshape", B=B, H_q=H_q, H_kv=H_kv, d=d, L_max=900, dtype=torch.bfloat16, seed=42)
    _run(oracle, w, [900, 333, 17][:B], 200)


def test_window_f32(oracle):
    w = inputs.custom("winf32", B=3, H_q=8, H_kv=2, d=64, L_max=400, dtype=torch.float32, seed=43)
    _run(oracle, w, [400, 65, 1], 70)


def test_window_covering_everything_equals_full_decode():
    w = inputs.custom("winfull", B=3, H_q=16, H_kv=4, d=128, L_max=700, dtype=torch.bfloat16, seed=44)
    x = inputs.make_inputs(w, lengths=[700, 3, 450])
    g = to_dev(x)
    a = gqa.decode(g["q"], g["k_cache"], g["v_cache"], g["lengths"], x["scale"])
    b = gqa.decode_window(g["q"], g["k_cache"], g["v_cache"], g["lengths"], 700, x["scale"])
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_window_full_size_ragged(oracle):
    """The ragged long-context batch with W = 4096, sampled sequences."""
    w = inputs.WORKLOADS["ragged_long_window4096"]
    x = inputs.make_inputs(w)
    g = to_dev(x)
    out = gqa.decode_window(g["q"], g["k_cache"], g["v_cache"], g["lengths"], w.window, x["scale"])
    torch.cuda.synchronize()
    lens = x["lengths"].tolist()
    bs = sorted({0, w.B - 1, int(np.argmin(lens)), int(np.argmax(lens))})
    for b in bs:
        ref = oracle.decode_window(x["q"][b:b + 1].double().numpy(), x["k_cache"][b:b + 1].double().numpy(),
                                   x["v_cache"][b:b + 1].double().numpy(), x["lengths"][b:b + 1].numpy(),
                                   w.window, x["scale"])
        assert float(np.max(np.abs(out[b].cpu().double().numpy() - ref[0]))) <= TOL[w.dtype], b

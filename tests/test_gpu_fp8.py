"""GPU parity of the FP8 (e4m3) cache: gqa_kv_append_fp8 bit for bit, and gqa_decode_fp8 /
gqa_decode_paged_fp8 against the oracle fed the dequantised values.

Cache rows past each sequence's length hold the NaN code, so a read past the length poisons
the output.  Lengths straddle the 256- and 128-row tiles of the kernel and its 8-row tail boxes.
"""
import numpy as np
import pytest
import torch

import grouped_query_attention_decode_b200 as gqa
from grouped_query_attention_decode_b200 import inputs

pytestmark = pytest.mark.gpu

TOL = 2e-3  # the bf16-cache tolerance, with the oracle fed the dequantised values


def _oracle_fp8(oracle, x, bs, window=0):
    """Oracle append (quantising) + decode for sequences bs; returns (codes K, codes V, lens, ref)."""
    kc = x["k_cache"][bs].numpy().copy()
    vc = x["v_cache"][bs].numpy().copy()
    lens = x["seq_lens_pre"][bs].numpy().copy()
    ks, vs = x["k_scale"].numpy(), x["v_scale"].numpy()
    st = oracle.kv_append_fp8(x["k_new"][bs].float().numpy(), x["v_new"][bs].float().numpy(),
                              kc, vc, ks, vs, lens)
    assert st == 0
    ref = oracle.decode_fp8(x["q"][bs].double().numpy(), kc, vc, ks, vs, lens, x["scale"], window=window)
    return kc, vc, lens, ref


def _step(oracle, w, lengths=None, window=0, bs=None):
    x = inputs.make_inputs(w, lengths=lengths, poison=True)
    dev = "cuda"
    kc, vc = x["k_cache"].to(dev), x["v_cache"].to(dev)
    ks, vs = x["k_scale"].to(dev), x["v_scale"].to(dev)
    lens = x["seq_lens_pre"].to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    gqa.kv_append_fp8(x["k_new"].to(dev), x["v_new"].to(dev), kc, vc, ks, vs, lens, status=status)
    out = gqa.decode_fp8(x["q"].to(dev), kc, vc, ks, vs, lens, x["scale"], window=window, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(lens.cpu(), x["lengths"])
    bs = list(range(w.B)) if bs is None else list(bs)
    kco, vco, _, ref = _oracle_fp8(oracle, x, bs, window)
    # the append's codes, bit for bit
    kh, vh = kc.cpu().numpy(), vc.cpu().numpy()
    for i, b in enumerate(bs):
        t = int(x["seq_lens_pre"][b])
        assert np.array_equal(kh[b, t], kco[i, t]) and np.array_equal(vh[b, t], vco[i, t])
    got = out[bs].cpu().double().numpy()
    assert np.isfinite(got).all()
    err = float(np.max(np.abs(got - ref)))
    assert err <= TOL, err
    return err


def _special_rows(shape, dtype, seed):
    """New rows with ties between codes, saturation, subnormal-range and signed-zero values."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g) * 40
    flat = x.view(-1)
    n = flat.numel()
    codes = torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).float()
    mids = (codes[:-1] + codes[1:]) / 2  # exact ties (scale 1)
    k = min(n // 4, mids.numel())
    flat[:k] = mids[:k] * torch.where(torch.arange(k) % 2 == 0, 1.0, -1.0)
    flat[k:k + 8] = torch.tensor([500.0, -500.0, 449.0, 464.0, -464.0, 1e-4, -0.0, 0.0])
    return x.to(dtype)


@pytest.mark.parametrize("new_dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_fp8_append_bit_exact(oracle, new_dtype):
    B, L, H_kv, d = 3, 40, 2, 128
    dev = "cuda"
    kn = _special_rows((B, H_kv, d), new_dtype, 1)
    vn = _special_rows((B, H_kv, d), new_dtype, 2)
    ks = torch.tensor([1.0, 0.37], dtype=torch.float32)
    vs = torch.tensor([0.5, 3.0], dtype=torch.float32)
    kc = torch.zeros((B, L, H_kv, d), dtype=torch.uint8)
    vc = torch.zeros_like(kc)
    lens = torch.tensor([0, 17, L], dtype=torch.int32)  # the last one is full: refused
    kcd, vcd, ld = kc.to(dev), vc.to(dev), lens.to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    gqa.kv_append_fp8(kn.to(dev), vn.to(dev), kcd, vcd, ks.to(dev), vs.to(dev), ld, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == gqa.STATUS_APPEND_OVERFLOW
    kco, vco, lo = kc.numpy().copy(), vc.numpy().copy(), lens.numpy().copy()
    assert oracle.kv_append_fp8(kn.float().numpy(), vn.float().numpy(), kco, vco, ks.numpy(), vs.numpy(), lo) == 1
    assert np.array_equal(ld.cpu().numpy(), lo)
    assert np.array_equal(kcd.cpu().numpy(), kco)
    assert np.array_equal(vcd.cpu().numpy(), vco)


@pytest.mark.parametrize("shape", [
    (4, 64, 8, 128), (3, 32, 8, 128), (3, 8, 8, 128), (2, 16, 1, 128), (2, 32, 1, 128),
    (2, 64, 1, 64), (3, 16, 4, 64), (2, 8, 2, 64), (2, 128, 2, 128),
], ids=lambda s: "B%d_Hq%d_Hkv%d_d%d" % s)
def test_fp8_decode_group_sizes(oracle, shape):
    B, H_q, H_kv, d = shape
    w = inputs.custom("fp8g", B=B, H_q=H_q, H_kv=H_kv, d=d, L_max=1100, kv_format="e4m3", seed=61)
    lengths = [1, 255, 256, 257, 520, 1100, 129, 700][:B]
    _step(oracle, w, lengths)


def test_fp8_decode_tile_edges(oracle):
    # lengths around the 256-row tile and the 8-row tail boxes, several sequences per CTA
    w = inputs.custom("fp8e", B=12, H_q=16, H_kv=4, d=128, L_max=1030, kv_format="e4m3", seed=62)
    _step(oracle, w, [1, 2, 7, 8, 9, 248, 255, 256, 257, 263, 512, 1030])


def test_fp8_decode_peaked_scores(oracle):
    # large q: a few rows dominate the softmax, the case that needs P's lower terms
    w = inputs.custom("fp8p", B=3, H_q=32, H_kv=4, d=128, L_max=900, kv_format="e4m3",
                      q_std=4.0, seed=63)
    _step(oracle, w, [900, 333, 17])


@pytest.mark.parametrize("window", [1, 100, 256, 4096])
def test_fp8_decode_window(oracle, window):
    w = inputs.custom("fp8w", B=4, H_q=32, H_kv=8, d=128, L_max=2000, kv_format="e4m3", seed=64)
    _step(oracle, w, [2000, 700, 256, 30], window=window)


def test_fp8_full_size_llama(oracle):
    w = inputs.WORKLOADS["llama2_70b_layer_fp8"]
    _step(oracle, w, bs=list(range(w.B)))


@pytest.mark.parametrize("page_size", [8, 16, 64, 256, 512])
def test_fp8_paged(oracle, page_size):
    w = inputs.custom("fp8pg", B=4, H_q=32, H_kv=8, d=128, L_max=1024, kv_format="e4m3", seed=65)
    x = inputs.make_inputs(w, lengths=[1, 300, 1000, 1024], poison=True)
    pg = inputs.make_paged(x, page_size)
    dev = "cuda"
    kp, vp, bt = pg["k_pool"].to(dev), pg["v_pool"].to(dev), pg["block_table"].to(dev)
    ks, vs = x["k_scale"].to(dev), x["v_scale"].to(dev)
    lens = x["seq_lens_pre"].to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    gqa.kv_append_paged_fp8(x["k_new"].to(dev), x["v_new"].to(dev), kp, vp, ks, vs, bt, lens, status=status)
    out = gqa.decode_paged_fp8(x["q"].to(dev), kp, vp, ks, vs, bt, lens, x["scale"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kpo, vpo = pg["k_pool"].numpy().copy(), pg["v_pool"].numpy().copy()
    lo = x["seq_lens_pre"].numpy().copy()
    bto = pg["block_table"].numpy()
    assert oracle.kv_append_paged_fp8(x["k_new"].float().numpy(), x["v_new"].float().numpy(), kpo, vpo,
                                      x["k_scale"].numpy(), x["v_scale"].numpy(), bto, lo) == 0
    assert np.array_equal(kp.cpu().numpy(), kpo) and np.array_equal(vp.cpu().numpy(), vpo)
    ref = oracle.decode_paged_fp8(x["q"].double().numpy(), kpo, vpo, x["k_scale"].numpy(),
                                  x["v_scale"].numpy(), bto, lo, x["scale"])
    err = float(np.max(np.abs(out.cpu().double().numpy() - ref)))
    assert err <= TOL, err


def test_fp8_rejects_bad_arguments():
    dev = "cuda"
    q = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device=dev)
    kc = torch.zeros((1, 64, 2, 128), dtype=torch.uint8, device=dev)
    lens = torch.ones(1, dtype=torch.int32, device=dev)
    sc = torch.ones(2, dtype=torch.float32, device=dev)
    lib = gqa.load_library()
    out = torch.empty((1, 8, 128), dtype=torch.float32, device=dev)
    ws = gqa.alloc_workspace_fp8(1, 8, 2, 128)
    args = lambda ksc: (gqa._ptr(q), gqa._ptr(kc), gqa._ptr(kc), ksc, gqa._ptr(sc), gqa._ptr(lens), 1, 8, 2,
                        128, 64, 0, 0.1, gqa._ptr(out), gqa._ptr(ws), ws.numel(), None, gqa._stream(None))
    assert lib.gqa_decode_fp8(*args(None)) == -1
    # the 16-bit entry points do not take the e4m3 type
    assert lib.gqa_decode(gqa._ptr(q), gqa._ptr(kc), gqa._ptr(kc), gqa._ptr(lens), 1, 8, 2, 128, 64, 0.1,
                          gqa.DTYPE_E4M3, gqa._ptr(out), gqa._ptr(ws), ws.numel(), None, gqa._stream(None)) == -5


@pytest.mark.parametrize("shape", [(4, 32, 4), (4, 16, 4), (3, 64, 4), (2, 64, 2)],
                         ids=lambda s: "B%d_Hq%d_Hkv%d" % s)
def test_fp8_many_tiles_per_cta(oracle, shape):
    # far more tiles than SMs: every CTA streams several tiles (the tile-alternating warpgroups
    # of the small-group kernels both work), cuts units into pieces and ends on partial tiles
    B, H_q, H_kv = shape
    w = inputs.custom("fp8m", B=B, H_q=H_q, H_kv=H_kv, d=128, L_max=12000, kv_format="e4m3",
                      q_std=2.0, seed=66)
    _step(oracle, w, [12000, 11111, 9000, 10001][:B])

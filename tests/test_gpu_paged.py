"""GPU parity of the paged cache (gqa_kv_append_paged + gqa_decode_paged) against the oracle.

The contiguous test caches are scattered into a pool of pages in a random order (with unused
NaN pages mixed in, and NaN in every row past each sequence's length), so a wrong page, a wrong
row within a page, or a read past the length shows up in the output.
"""
import numpy as np
import pytest
import torch

import grouped_query_attention_decode_b200 as gqa
import oracle as oracle_mod
from gpu_helpers import TOL
from grouped_query_attention_decode_b200 import inputs

pytestmark = pytest.mark.gpu


def _step(oracle, w, lengths, page_size, bs=None):
    x = inputs.make_inputs(w, lengths=lengths, poison=True)
    pg = inputs.make_paged(x, page_size)
    dev = "cuda"
    kp, vp, bt = pg["k_pool"].to(dev), pg["v_pool"].to(dev), pg["block_table"].to(dev)
    lens = x["seq_lens_pre"].to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    gqa.kv_append_paged(x["k_new"].to(dev), x["v_new"].to(dev), kp, vp, bt, lens, status=status)
    out = gqa.decode_paged(x["q"].to(dev), kp, vp, bt, lens, x["scale"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(lens.cpu(), x["lengths"])
    assert torch.isfinite(out).all()
    # oracle: paged append + paged decode on float64 copies of the same pools
    kpo, vpo = pg["k_pool"].double().numpy().copy(), pg["v_pool"].double().numpy().copy()
    lo = x["seq_lens_pre"].numpy().copy()
    bto = pg["block_table"].numpy()
    assert oracle.kv_append_paged(x["k_new"].double().numpy(), x["v_new"].double().numpy(), kpo, vpo, bto, lo) == 0
    bs = list(range(w.B)) if bs is None else bs
    ref = oracle.decode_paged(x["q"][bs].double().numpy(), kpo, vpo, bto[bs], lo[bs], x["scale"])
    got = out[bs].cpu().double().numpy()
    err = float(np.max(np.abs(got - ref)))
    assert err <= TOL[w.dtype], err
    # the paged append wrote exactly the new rows (bit exact)
    kp_h = kp.cpu()
    for b in bs:
        t = int(x["seq_lens_pre"][b])
        page = int(bt[b, t // page_size])
        assert torch.equal(kp_h[page, t % page_size], x["k_new"][b])


@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
def test_paged_bf16_page_sizes(oracle, page_size):
    w = inputs.custom("paged", B=4, H_q=32, H_kv=8, d=128, L_max=1024, dtype=torch.bfloat16, seed=51)
    _step(oracle, w, [1, 129, 1000, 1024], page_size)


@pytest.mark.parametrize("shape", [(3, 64, 1, 64), (2, 16, 16, 64), (2, 24, 2, 128)],
                         ids=lambda s: "B%d_Hq%d_Hkv%d_d%d" % s)
def test_paged_group_sizes(oracle, shape):
    B, H_q, H_kv, d = shape
    w = inputs.custom("pagedg", B=B, H_q=H_q, H_kv=H_kv, d=d, L_max=512, dtype=torch.bfloat16, seed=52)
    _step(oracle, w, [512, 17, 300][:B], 16)


@pytest.mark.parametrize("page_size", [8, 64, 256, 512])
def test_paged_d64_256_row_tiles(oracle, page_size):
    # 64-wide heads in groups of up to 8 take 256-row tiles: pages smaller than, equal to and
    # larger than a tile
    w = inputs.custom("paged64", B=3, H_q=16, H_kv=2, d=64, L_max=1024, dtype=torch.bfloat16, seed=56)
    _step(oracle, w, [1024, 257, 40], page_size)


@pytest.mark.parametrize("page_size", [8, 24])
def test_paged_f32(oracle, page_size):
    w = inputs.custom("pagedf", B=3, H_q=8, H_kv=2, d=64, L_max=240, dtype=torch.float32, seed=53)
    _step(oracle, w, [240, 65, 9], page_size)


def test_paged_full_size_llama(oracle):
    w = inputs.WORKLOADS["llama2_70b_layer_paged16"]
    _step(oracle, w, None, w.page_size, bs=[0, 7, 15])


def test_paged_bad_page_is_reported(oracle):
    w = inputs.custom("pagedbad", B=2, H_q=16, H_kv=4, d=128, L_max=256, dtype=torch.bfloat16, seed=54)
    x = inputs.make_inputs(w, lengths=[256, 40])
    pg = inputs.make_paged(x, 32)
    bt = pg["block_table"].clone()
    bt[1, 0] = 10_000  # no such page
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gqa.decode_paged(x["q"].cuda(), pg["k_pool"].cuda(), pg["v_pool"].cuda(), bt.cuda(),
                           x["lengths"].cuda(), x["scale"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & gqa.STATUS_PAGE_RANGE
    # the oracle reports the same entry; the sequence with a valid table still matches it
    ref, st = oracle.decode_paged(x["q"].double().numpy(), pg["k_pool"].double().numpy(),
                                  pg["v_pool"].double().numpy(), bt.numpy(), x["lengths"].numpy(),
                                  x["scale"], return_status=True)
    assert st & oracle_mod.PAGE_RANGE
    assert float(np.max(np.abs(out[0].cpu().double().numpy() - ref[0]))) <= TOL[w.dtype]


def test_paged_rejects_unsupported_page_size():
    w = inputs.custom("pagedrej", B=1, H_q=8, H_kv=2, d=64, L_max=96, dtype=torch.bfloat16, seed=55)
    x = inputs.make_inputs(w, lengths=[96])
    pg = inputs.make_paged(x, 24)  # 24 neither divides the 256-row tile nor is a multiple of it
    with pytest.raises(gqa.GQAError):
        gqa.decode_paged(x["q"].cuda(), pg["k_pool"].cuda(), pg["v_pool"].cuda(),
                         pg["block_table"].cuda(), x["lengths"].cuda(), x["scale"])

"""GPU parity of gqa_kv_append_decode, the append and the decode of one step in one launch.

It must give what gqa_kv_append followed by gqa_decode gives, bit for bit (outputs and cache
bytes), and match the oracle's append + decode within the bf16 tolerance; the input lengths
are only read and the new ones land in the second array.  Cache rows past each sequence's
length are NaN, so a read past the length shows up in the output.
"""
import numpy as np
import pytest
import torch

import grouped_query_attention_decode_b200 as gqa
from gpu_helpers import TOL, max_err, oracle_step, workload
from grouped_query_attention_decode_b200 import inputs

pytestmark = pytest.mark.gpu


def _both(x):
    """(fused out, fused caches, lens_in after, lens_out, status) and the two-call
    (out, caches, lens, status) on separate copies of the same device inputs."""
    dev = "cuda"
    q, kn, vn = x["q"].to(dev), x["k_new"].to(dev), x["v_new"].to(dev)
    k1, v1 = x["k_cache"].to(dev), x["v_cache"].to(dev)
    k2, v2 = k1.clone(), v1.clone()
    lens_in = x["seq_lens_pre"].to(dev)
    lens_out = torch.full_like(lens_in, -7)
    st1 = torch.zeros(1, dtype=torch.int32, device=dev)
    out1 = gqa.kv_append_decode(q, kn, vn, k1, v1, lens_in, lens_out, x["scale"], status=st1)
    lens2 = x["seq_lens_pre"].to(dev)
    st2 = torch.zeros(1, dtype=torch.int32, device=dev)
    gqa.kv_append(kn, vn, k2, v2, lens2, status=st2)
    out2 = gqa.decode(q, k2, v2, lens2, x["scale"], status=st2)
    torch.cuda.synchronize()
    return (out1, (k1, v1), lens_in, lens_out, int(st1.item())), (out2, (k2, v2), lens2, int(st2.item()))


def _check(oracle, w, lengths=None, poison=True):
    x = inputs.make_inputs(w, lengths=lengths, poison=poison)
    (out1, c1, lens_in, lens_out, st1), (out2, c2, lens2, st2) = _both(x)
    assert st1 == 0 and st2 == 0
    assert torch.equal(lens_in.cpu(), x["seq_lens_pre"]), "the input lengths are only read"
    assert torch.equal(lens_out.cpu(), x["lengths"]) and torch.equal(lens2.cpu(), x["lengths"])
    assert torch.equal(out1, out2), "fused and two-call outputs differ"
    for a, b in zip(c1, c2):
        # NaN-poisoned rows compare equal as bytes
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), "cache bytes differ"
    ref = oracle_step(oracle, x, None)
    err = max_err(out1, ref)
    assert err <= TOL[w.dtype], f"{w.name}: max abs error {err}"


SHAPES = [
    (3, 8, 8, 128),    # MHA
    (2, 16, 2, 128),   # r = 8
    (2, 32, 2, 64),    # r = 16
    (2, 32, 1, 128),   # r = 32
    (2, 64, 1, 64),    # r = 64
    (1, 128, 1, 128),  # r = 128: two head blocks share the appended row
    (2, 24, 2, 128),   # r = 12
    (3, 16, 4, 64),    # r = 4 at d = 64: 256-row tiles
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B%d_Hq%d_Hkv%d_d%d" % s)
def test_fused_small(oracle, shape):
    B, H_q, H_kv, d = shape
    w = inputs.custom(f"fused_{B}_{H_q}_{H_kv}_{d}", B=B, H_q=H_q, H_kv=H_kv, d=d, L_max=1100,
                      dtype=torch.bfloat16, q_std=0.5, kv_std=1.0, seed=300 + H_q + H_kv + d)
    choices = [1, 7, 8, 9, 127, 128, 129, 255, 256, 257, 1000, 1100]
    lengths = [choices[(i * 5 + H_kv + 3) % len(choices)] for i in range(B)]
    _check(oracle, w, lengths=lengths)


def test_fused_many_short_sequences(oracle):
    # more units than CTAs, one partial tile each: the appended row is in every unit's only tile
    w = inputs.custom("fused_short", B=300, H_q=16, H_kv=4, d=128, L_max=40, dtype=torch.bfloat16, seed=31)
    _check(oracle, w, lengths=[1 + (7 * i) % 40 for i in range(300)])


@pytest.mark.parametrize("name", ["llama2_70b_layer", "ragged_long", "mqa_long"])
def test_fused_full_size(oracle, name):
    _check(oracle, workload(name), poison=False)


def test_fused_full_cache_and_out_of_range_lengths(oracle):
    w = inputs.custom("fused_edge", B=4, H_q=16, H_kv=2, d=128, L_max=256, dtype=torch.bfloat16, seed=33)
    x = inputs.make_inputs(w, lengths=[256, 10, 256, 1])
    dev = "cuda"
    lens_in = torch.tensor([256, 9, 300, -1], dtype=torch.int32, device=dev)  # full, ok, past L_max, negative
    lens_out = torch.zeros_like(lens_in)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    kc, vc = x["k_cache"].to(dev), x["v_cache"].to(dev)
    k0 = kc.clone()
    out = gqa.kv_append_decode(x["q"].to(dev), x["k_new"].to(dev), x["v_new"].to(dev), kc, vc, lens_in,
                               lens_out, x["scale"], status=status)
    torch.cuda.synchronize()
    st = int(status.item())
    assert st & gqa.STATUS_APPEND_OVERFLOW and st & gqa.STATUS_SEQLEN_RANGE
    assert lens_out.cpu().tolist() == [256, 10, 300, -1]
    # nothing was appended to the full sequence or the out-of-range ones; sequence 1 got row 9
    for b in (0, 2, 3):
        assert torch.equal(kc[b], k0[b])
    assert torch.equal(kc[1, 9].cpu(), x["k_new"][1])
    assert torch.equal(out[2], torch.zeros_like(out[2])) and torch.equal(out[3], torch.zeros_like(out[3]))
    # sequence 0 attends all 256 rows, sequence 1 its 10 (the appended one included)
    xs = dict(x)
    xs["k_cache"], xs["v_cache"] = kc.cpu(), vc.cpu()
    xs["lengths"] = torch.tensor([256, 10, 0, 0], dtype=torch.int32)
    ref = oracle_step(oracle, xs, [0, 1], append=False)
    assert max_err(out, ref) <= TOL[w.dtype]


def test_fused_repeated_steps_grow_the_sequences(oracle):
    """A decode loop: lengths ping-pong between two arrays, each step appends one row."""
    w = inputs.custom("fused_loop", B=3, H_q=32, H_kv=4, d=128, L_max=400, dtype=torch.bfloat16, seed=34)
    x = inputs.make_inputs(w, lengths=[100, 250, 1])
    dev = "cuda"
    g = torch.Generator().manual_seed(5)
    kc, vc = x["k_cache"].to(dev), x["v_cache"].to(dev)
    lens = [x["seq_lens_pre"].to(dev), torch.zeros(3, dtype=torch.int32, device=dev)]
    kh, vh = x["k_cache"].double().numpy().copy(), x["v_cache"].double().numpy().copy()
    lh = x["seq_lens_pre"].numpy().copy()
    ws = gqa.alloc_workspace(w.B, w.H_q, w.H_kv, w.d, w.dtype)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for s in range(5):
        q = torch.randn((3, 32, 128), generator=g).to(torch.bfloat16)
        kn = torch.randn((3, 4, 128), generator=g).to(torch.bfloat16)
        vn = torch.randn((3, 4, 128), generator=g).to(torch.bfloat16)
        out = gqa.kv_append_decode(q.to(dev), kn.to(dev), vn.to(dev), kc, vc, lens[s & 1], lens[(s + 1) & 1],
                                   x["scale"], workspace=ws, status=status)
        oracle.kv_append(kn.double().numpy(), vn.double().numpy(), kh, vh, lh)
        ref = oracle.decode(q.double().numpy(), kh, vh, lh, x["scale"])
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert lens[(s + 1) & 1].cpu().tolist() == lh.tolist()
        assert float(np.max(np.abs(out.cpu().double().numpy() - ref))) <= TOL[w.dtype]

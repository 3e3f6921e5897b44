"""GPU parity of several query tokens per sequence (gqa_kv_append_multi + gqa_decode_multi)
against the oracle: token j of Q attends rows [0, n - Q + 1 + j) (speculative verification,
causal among the drafts).  Rows past n are NaN."""
import numpy as np
import pytest
import torch

import grouped_query_attention_decode_b200 as gqa
from gpu_helpers import TOL, to_dev
from grouped_query_attention_decode_b200 import inputs

pytestmark = pytest.mark.gpu


def _step(oracle, w, lengths, bs=None):
    x = inputs.make_inputs(w, lengths=lengths, poison=True)
    g = to_dev(x)
    lens = g["seq_lens_pre"].clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gqa.kv_append_multi(g["k_new"], g["v_new"], g["k_cache"], g["v_cache"], lens, status=status)
    out = gqa.decode_multi(g["q"], g["k_cache"], g["v_cache"], lens, x["scale"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(lens.cpu(), x["lengths"])
    assert torch.isfinite(out).all()
    bs = list(range(w.B)) if bs is None else bs
    kc = x["k_cache"][bs].double().numpy().copy()
    vc = x["v_cache"][bs].double().numpy().copy()
    lo = x["seq_lens_pre"][bs].numpy().copy()
    for j in range(w.queries):
        oracle.kv_append(x["k_new"][bs, j].double().numpy(), x["v_new"][bs, j].double().numpy(), kc, vc, lo)
    ref = oracle.decode_multi(x["q"][bs].double().numpy(), kc, vc, lo, x["scale"])
    err = float(np.max(np.abs(out[bs].cpu().double().numpy() - ref)))
    assert err <= TOL[w.dtype], err
    # the appended rows are the new ones, bit for bit
    kg = g["k_cache"].cpu()
    for b in bs:
        t = int(x["seq_lens_pre"][b])
        assert torch.equal(kg[b, t:t + w.queries], x["k_new"][b])


@pytest.mark.parametrize("Q", [2, 3, 4, 8])
def test_multi_bf16(oracle, Q):
    w = inputs.custom("multi", B=4, H_q=32, H_kv=8, d=128, L_max=700, dtype=torch.bfloat16,
                      seed=60 + Q, queries=Q)
    _step(oracle, w, [Q, Q + 1, 129, 700])


@pytest.mark.parametrize("shape", [(2, 16, 16, 64, 4), (2, 32, 1, 128, 2), (2, 64, 1, 64, 2),
                                   (1, 128, 1, 128, 4)], ids=lambda s: "B%d_Hq%d_Hkv%d_d%d_Q%d" % s)
def test_multi_group_sizes(oracle, shape):
    B, H_q, H_kv, d, Q = shape
    w = inputs.custom("multig", B=B, H_q=H_q, H_kv=H_kv, d=d, L_max=400, dtype=torch.bfloat16,
                      seed=70, queries=Q)
    _step(oracle, w, [400, 130][:B])


def test_multi_f32(oracle):
    w = inputs.custom("multif", B=3, H_q=8, H_kv=2, d=64, L_max=200, dtype=torch.float32, seed=71,
                      queries=3)
    _step(oracle, w, [3, 65, 200])


def test_multi_one_token_is_the_plain_decode():
    w = inputs.custom("multi1", B=3, H_q=16, H_kv=4, d=128, L_max=500, dtype=torch.bfloat16, seed=72)
    x = inputs.make_inputs(w, lengths=[500, 1, 260])
    g = to_dev(x)
    a = gqa.decode(g["q"], g["k_cache"], g["v_cache"], g["lengths"], x["scale"])
    b = gqa.decode_multi(g["q"].unsqueeze(1).contiguous(), g["k_cache"], g["v_cache"], g["lengths"], x["scale"])
    torch.cuda.synchronize()
    assert torch.equal(a, b[:, 0])


def test_multi_too_short_is_reported():
    w = inputs.custom("multishort", B=2, H_q=16, H_kv=4, d=128, L_max=64, dtype=torch.bfloat16,
                      seed=73, queries=4)
    x = inputs.make_inputs(w, lengths=[64, 10])
    g = to_dev(x)
    lens = torch.tensor([64, 3], dtype=torch.int32, device="cuda")  # 3 < Q
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gqa.decode_multi(g["q"], g["k_cache"], g["v_cache"], lens, x["scale"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & gqa.STATUS_SEQLEN_RANGE
    assert torch.equal(out[1].cpu(), torch.zeros_like(out[1].cpu()))


def test_multi_full_size(oracle):
    w = inputs.WORKLOADS["llama2_70b_layer_spec4"]
    _step(oracle, w, None, bs=list(range(w.B)))

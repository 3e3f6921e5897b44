"""GPU parity where the work partition cuts units into many pieces.

The split kernels give every CTA an equal run of tiles; a unit (sequence, key/value head, head
block) longer than a run is cut into pieces held by consecutive CTAs, whose partial results are
merged by the CTA that takes the unit's last ticket.  These cases stress that path: one unit
cut into a piece per CTA, ranges that hold a partial piece at both ends and whole units between,
and the same for the FP8 kernel.  Outputs must match the oracle and be bit-identical across
calls (the merge order does not depend on which CTA finishes last).
"""
import numpy as np
import pytest
import torch

import grouped_query_attention_decode_b200 as gqa
from gpu_helpers import TOL, max_err, oracle_step, run_step
from grouped_query_attention_decode_b200 import inputs

pytestmark = pytest.mark.gpu


def _check_twice(oracle, w, lengths):
    x = inputs.make_inputs(w, lengths=lengths, poison=True)
    out, lens, status, _ = run_step(x)
    assert status == 0, f"device status {status}"
    assert torch.equal(lens.cpu(), x["lengths"])
    assert torch.isfinite(out).all()
    err = max_err(out, oracle_step(oracle, x))
    assert err <= TOL[w.dtype], f"{w.name}: max abs error {err}"
    again, _, status2, _ = run_step(x)
    assert status2 == 0
    assert torch.equal(out, again)


def test_one_unit_cut_into_a_piece_per_cta(oracle):
    # 1 sequence x 1 key/value head: 313 tiles of 128 rows, so every CTA holds a piece of it
    w = inputs.custom("pieces_one", B=1, H_q=8, H_kv=1, d=128, L_max=40000, dtype=torch.bfloat16,
                      q_std=1.0, kv_std=1.0, seed=81)
    _check_twice(oracle, w, [40000])


def test_long_unit_beside_short_ones(oracle):
    # one long unit cut into many pieces, next to units that fit in one CTA's range
    w = inputs.custom("pieces_mix", B=4, H_q=16, H_kv=2, d=64, L_max=30000, dtype=torch.bfloat16,
                      seed=82)
    _check_twice(oracle, w, [30000, 5, 129, 3000])


def test_ranges_with_whole_units_between_partial_ones(oracle):
    # 128 units of 3 tiles over 148 CTAs: most ranges start and end inside a unit and hold a
    # whole unit or none between, so a CTA hands over two pieces and merges what it completes
    w = inputs.custom("pieces_between", B=64, H_q=16, H_kv=2, d=128, L_max=300, dtype=torch.bfloat16,
                      seed=83)
    rng = np.random.default_rng(83)
    _check_twice(oracle, w, rng.integers(257, 301, size=64).tolist())


def _fp8_step(x, dev="cuda"):
    kc, vc = x["k_cache"].to(dev), x["v_cache"].to(dev)
    ks, vs = x["k_scale"].to(dev), x["v_scale"].to(dev)
    lens = x["seq_lens_pre"].to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    gqa.kv_append_fp8(x["k_new"].to(dev), x["v_new"].to(dev), kc, vc, ks, vs, lens, status=status)
    out = gqa.decode_fp8(x["q"].to(dev), kc, vc, ks, vs, lens, x["scale"], status=status)
    torch.cuda.synchronize()
    return out, int(status.item())


def test_fp8_one_unit_cut_into_a_piece_per_cta(oracle):
    w = inputs.custom("pieces_fp8", B=1, H_q=8, H_kv=1, d=128, L_max=50000, kv_format="e4m3",
                      q_std=2.0, seed=84)
    x = inputs.make_inputs(w, lengths=[50000], poison=True)
    out, status = _fp8_step(x)
    assert status == 0, f"device status {status}"
    kh, vh = x["k_cache"].numpy().copy(), x["v_cache"].numpy().copy()
    lh = x["seq_lens_pre"].numpy().copy()
    assert oracle.kv_append_fp8(x["k_new"].float().numpy(), x["v_new"].float().numpy(), kh, vh,
                                x["k_scale"].numpy(), x["v_scale"].numpy(), lh) == 0
    ref = oracle.decode_fp8(x["q"].double().numpy(), kh, vh, x["k_scale"].numpy(), x["v_scale"].numpy(),
                            lh, x["scale"])
    err = float(np.max(np.abs(out.cpu().double().numpy() - ref)))
    assert err <= 2e-3, err
    again, status2 = _fp8_step(x)
    assert status2 == 0 and torch.equal(out, again)

"""The pieces of a split sequence are merged inside the split kernel through per-unit counters
in the workspace (0 between calls).  These tests reuse one workspace across calls whose
partitions differ, and recover from a timed-out call (which can leave counters set)."""
import numpy as np
import pytest
import torch

import grouped_query_attention_decode_b200 as gqa
from gpu_helpers import TOL, max_err, oracle_step, to_dev
from grouped_query_attention_decode_b200 import inputs

pytestmark = pytest.mark.gpu


def _case(seed, lengths, H_q=24, H_kv=8):
    # r = 3 columns per unit (an odd slot size), long sequences: units cut into several pieces
    w = inputs.custom("merge", B=len(lengths), H_q=H_q, H_kv=H_kv, d=128, L_max=9000, seed=seed)
    return w, inputs.make_inputs(w, lengths=lengths)


def test_one_workspace_many_calls(oracle):
    ws = None
    for seed, lengths in [(71, [9000, 5000, 1]), (72, [300, 8999, 4096]), (73, [9000, 9000, 9000]),
                          (74, [0, 7000, 129])]:
        w, x = _case(seed, lengths)
        if ws is None:
            ws = gqa.alloc_workspace(w.B, w.H_q, w.H_kv, w.d, w.dtype)
        g = to_dev(x)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = gqa.decode(g["q"], g["k_cache"], g["v_cache"], g["lengths"], x["scale"], workspace=ws, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref = oracle_step(oracle, x, append=False)
        assert max_err(out, ref) <= TOL[torch.bfloat16]
    # every call left the counters at zero
    off = 0  # the per-unit counters open the workspace
    units = w.B * w.H_kv  # rb = r = 3 columns: one unit per (sequence, kv head)
    counters = ws[off:off + units * 4 * 4].view(torch.int32)
    assert int(counters.abs().sum()) == 0


def test_rezeroed_workspace_after_timeout(oracle):
    w, x = _case(75, [9000, 8000, 7000])
    g = to_dev(x)
    ws = gqa.alloc_workspace(w.B, w.H_q, w.H_kv, w.d, w.dtype)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gqa.set_wait_timeout_ns(1)
    try:
        gqa.decode(g["q"], g["k_cache"], g["v_cache"], g["lengths"], x["scale"], workspace=ws, status=status)
        torch.cuda.synchronize()
    finally:
        gqa.set_wait_timeout_ns(0)
    assert int(status.item()) & gqa.STATUS_WAIT_TIMEOUT
    ws.zero_()  # the documented recovery: zero the workspace again
    status.zero_()
    out = gqa.decode(g["q"], g["k_cache"], g["v_cache"], g["lengths"], x["scale"], workspace=ws, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert max_err(out, oracle_step(oracle, x, append=False)) <= TOL[torch.bfloat16]


def test_noalloc_recovers_after_timeout(oracle):
    # gqa_decode_noalloc clears its own counters before every call
    w, x = _case(76, [9000, 6000, 8500])
    g = to_dev(x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gqa.set_wait_timeout_ns(1)
    try:
        gqa.decode_noalloc(g["q"], g["k_cache"], g["v_cache"], g["lengths"], x["scale"], status=status)
        torch.cuda.synchronize()
    finally:
        gqa.set_wait_timeout_ns(0)
    assert int(status.item()) & gqa.STATUS_WAIT_TIMEOUT
    status.zero_()
    out = gqa.decode_noalloc(g["q"], g["k_cache"], g["v_cache"], g["lengths"], x["scale"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert max_err(out, oracle_step(oracle, x, append=False)) <= TOL[torch.bfloat16]

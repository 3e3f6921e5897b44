"""GPU: one decode workspace reused across calls whose partitions differ.

The workspace keeps per-unit counters that every call leaves at zero again; a call must not
depend on what an earlier call on the same workspace did.  The output must match the oracle
for: the same lengths twice, other lengths (another partition of the tile line), another
geometry on the same workspace, a windowed call after a full one, and the fused append after a
decode.
"""
import pytest
import torch

import grouped_query_attention_decode_b200 as gqa
from gpu_helpers import TOL, max_err, oracle_step, to_dev
from grouped_query_attention_decode_b200 import inputs

pytestmark = pytest.mark.gpu


def _decode(oracle, x, ws, window=0):
    # decode only, over the rows the caches hold (rows from seq_lens_pre on are NaN)
    x = dict(x, lengths=x["seq_lens_pre"])
    g = to_dev(x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if window:
        out = gqa.decode_window(g["q"], g["k_cache"], g["v_cache"], g["lengths"], window, x["scale"],
                                workspace=ws, status=status)
    else:
        out = gqa.decode(g["q"], g["k_cache"], g["v_cache"], g["lengths"], x["scale"], workspace=ws,
                         status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    assert torch.isfinite(out).all()
    if not window:
        err = max_err(out, oracle_step(oracle, x, append=False))
        assert err <= TOL[torch.bfloat16], f"max abs error {err}"
    return out


def _shape(seed, H_kv=4, d=128):
    return inputs.custom("reuse", B=3, H_q=16, H_kv=H_kv, d=d, L_max=1024, dtype=torch.bfloat16, seed=seed)


@pytest.mark.parametrize("d", [128, 64])
def test_same_and_other_partitions(oracle, d):
    w = _shape(71, d=d)
    ws = gqa.alloc_workspace(w.B, w.H_q, w.H_kv, w.d, w.dtype)
    xa = inputs.make_inputs(w, lengths=[1024, 513, 200], poison=True)
    xb = inputs.make_inputs(w, lengths=[100, 1000, 700], poison=True)
    first = _decode(oracle, xa, ws)
    again = _decode(oracle, xa, ws)
    assert torch.equal(first, again), "the same call on a used workspace changed its output"
    _decode(oracle, xb, ws)           # another partition
    _decode(oracle, xb, ws)
    _decode(oracle, xa, ws)


def test_other_geometry_same_workspace(oracle):
    w = _shape(72)
    w2 = _shape(73, H_kv=2)
    n = max(gqa.workspace_size(v.B, v.H_q, v.H_kv, v.d, v.dtype) for v in (w, w2))
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    _decode(oracle, inputs.make_inputs(w, lengths=[1024, 1024, 1024], poison=True), ws)
    # another geometry on the same workspace
    x2 = inputs.make_inputs(w2, lengths=[1024, 1024, 1024], poison=True)
    _decode(oracle, x2, ws)
    _decode(oracle, x2, ws)


def test_window_after_full(oracle):
    w = _shape(74)
    ws = gqa.alloc_workspace(w.B, w.H_q, w.H_kv, w.d, w.dtype)
    x = inputs.make_inputs(w, lengths=[1024, 900, 600], poison=True)
    _decode(oracle, x, ws)
    # the windowed call twice on the used workspace: the same output both times (the windowed
    # path's own parity against the oracle is covered elsewhere)
    a = _decode(oracle, x, ws, window=256)
    b = _decode(oracle, x, ws, window=256)
    assert torch.equal(a, b)


def test_fused_append_after_decode(oracle):
    w = _shape(75)
    ws = gqa.alloc_workspace(w.B, w.H_q, w.H_kv, w.d, w.dtype)
    x = inputs.make_inputs(w, lengths=[1024, 257, 129], poison=True)
    # decode over the lengths after the append, on the caches before it (the same partition as
    # the fused launch below), then the fused launch twice on that workspace
    g = to_dev(x)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gqa.decode(g["q"], g["k_cache"], g["v_cache"], g["lengths"], x["scale"], workspace=ws, status=status)
    lens_out = torch.full_like(g["seq_lens_pre"], -7)
    for _ in range(2):
        kc, vc = g["k_cache"].clone(), g["v_cache"].clone()
        out = gqa.kv_append_decode(g["q"], g["k_new"], g["v_new"], kc, vc, g["seq_lens_pre"], lens_out,
                                   x["scale"], workspace=ws, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(lens_out.cpu(), x["lengths"])
        err = max_err(out, oracle_step(oracle, x))
        assert err <= TOL[torch.bfloat16], f"max abs error {err}"

"""Failure detection on the GPU without faulting it.

Every pipeline wait inside the decode kernel is bounded.  With a 1 ns limit the waits run out at
once; the kernel must then report GQA_STATUS_WAIT_TIMEOUT, wait for its own copies and tensor-core
work in flight, free its tensor memory and return, leaving the context usable: the next call,
with the default limit, must be correct.  Host-side refusals (bad sizes) are covered on the CPU
in test_abi.py; device-side range checks in test_gpu_parity.py.
"""
import pytest
import torch

import grouped_query_attention_decode_b200 as gqa
from gpu_helpers import TOL, max_err, oracle_step, to_dev
from grouped_query_attention_decode_b200 import inputs

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_the_context_recovers(oracle):
    w = inputs.custom("timeout", B=4, H_q=32, H_kv=8, d=128, L_max=4096, seed=31, length=4096)
    x = inputs.make_inputs(w)
    g = to_dev(x)
    lens = g["lengths"]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gqa.set_wait_timeout_ns(1)
    try:
        gqa.decode(g["q"], g["k_cache"], g["v_cache"], lens, x["scale"], status=status)
        torch.cuda.synchronize()
        st = int(status.item())
    finally:
        gqa.set_wait_timeout_ns(0)
    assert st & gqa.STATUS_WAIT_TIMEOUT
    status.zero_()
    out = gqa.decode(g["q"], g["k_cache"], g["v_cache"], lens, x["scale"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle_step(oracle, x, [0, 3], append=False)
    assert max_err(out, ref) <= TOL[torch.bfloat16]

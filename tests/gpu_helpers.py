"""Shared plumbing of the GPU parity tests: run one append + decode step through the C ABI and
evaluate the CPU oracle on the same (already rounded) values."""
from __future__ import annotations

import numpy as np
import torch

import grouped_query_attention_decode_b200 as gqa
from grouped_query_attention_decode_b200 import inputs

TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-3}


def to_dev(x: dict, dev="cuda") -> dict:
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def run_step(x: dict, append: bool = True, dev="cuda"):
    """Append (optional) then decode on the GPU.  Returns (out, seq_lens after, status, device
    tensors)."""
    g = to_dev(x, dev)
    lens = g["seq_lens_pre"].clone() if append else g["lengths"].clone()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    if append:
        gqa.kv_append(g["k_new"], g["v_new"], g["k_cache"], g["v_cache"], lens, status=status)
    out = gqa.decode(g["q"], g["k_cache"], g["v_cache"], lens, x["scale"], status=status)
    torch.cuda.synchronize()
    return out, lens, int(status.item()), g


def oracle_step(o, x: dict, bs=None, append: bool = True):
    """Oracle output for sequences ``bs`` (all when None), computed one sequence at a time on
    float64 copies of the same values."""
    B = x["q"].shape[0]
    bs = list(range(B)) if bs is None else list(bs)
    res = {}
    for b in bs:
        q = x["q"][b:b + 1].double().numpy()
        kc = x["k_cache"][b:b + 1].double().numpy().copy()
        vc = x["v_cache"][b:b + 1].double().numpy().copy()
        if append:
            lens = x["seq_lens_pre"][b:b + 1].numpy().copy()
            o.kv_append(x["k_new"][b:b + 1].double().numpy(), x["v_new"][b:b + 1].double().numpy(),
                        kc, vc, lens)
        else:
            lens = x["lengths"][b:b + 1].numpy().copy()
        res[b] = o.decode(q, kc, vc, lens, x["scale"])[0]
    return res


def max_err(out: torch.Tensor, ref: dict) -> float:
    o = out.detach().cpu().double().numpy()
    return max(float(np.max(np.abs(o[b] - r))) for b, r in ref.items())


def workload(name):
    return inputs.WORKLOADS[name]

"""GPU parity: the CUDA path through the C ABI against the CPU oracle, element by element.

Small cases and the full-size workloads (the shapes the benchmark times, launched the same
way) are checked on every output.  Tolerances: max abs
error 1e-5 for float32 inputs, 2e-3 for bf16 caches (fp32 accumulation; the oracle gets the
same bf16-rounded values).  The append is checked bit for bit.  Cache rows past each sequence's
length are NaN in these tests, so any read past the length shows up as NaN in the output.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import TOL, max_err, oracle_step, run_step, workload
from grouped_query_attention_decode_b200 import inputs

pytestmark = pytest.mark.gpu


def _check(oracle, w, lengths=None, bs=None, poison=True):
    x = inputs.make_inputs(w, lengths=lengths, poison=poison)
    out, lens, status, _ = run_step(x)
    assert status == 0, f"device status {status}"
    assert torch.equal(lens.cpu(), x["lengths"])
    ref = oracle_step(oracle, x, bs)
    err = max_err(out, ref)
    assert err <= TOL[w.dtype], f"{w.name}: max abs error {err}"
    assert torch.isfinite(out).all()
    return err


def test_tiny_fp32(oracle):
    _check(oracle, workload("tiny_fp32"))


@pytest.mark.parametrize("name", ["llama2_70b_layer", "t5xxl_g64_mha", "t5xxl_g8", "t5xxl_g1_mqa",
                                  "mqa_long", "ragged_long"])
def test_full_size_workloads(oracle, name):
    # every output of every sequence, at the sizes and in the launch configuration the
    # benchmark times
    w = workload(name)
    x = inputs.make_inputs(w, poison=False)
    out, lens, status, _ = run_step(x)
    assert status == 0, f"device status {status}"
    assert torch.equal(lens.cpu(), x["lengths"])
    assert torch.isfinite(out).all()
    ref = oracle_step(oracle, x, None)
    assert len(ref) == w.B
    err = max_err(out, ref)
    assert err <= TOL[w.dtype], f"{name}: max abs error {err}"


# group sizes 1..128 (64 and 128 = two and four blocks of 32 query heads), both head dims, lengths spanning
# several 128-row tiles with ragged tails (1, 7, 8, 9, 127, 128, 129, 255, 256, 257, 1000)
BF16_SHAPES = [
    (3, 8, 8, 128),    # MHA
    (3, 16, 4, 128),   # r = 4
    (2, 16, 2, 128),   # r = 8
    (2, 32, 2, 64),    # r = 16
    (2, 32, 1, 128),   # r = 32, MQA
    (2, 64, 1, 64),    # r = 64, MQA
    (1, 128, 1, 128),  # r = 128: two head blocks
    (2, 96, 2, 64),    # r = 48: padded to 64
    (2, 24, 2, 128),   # r = 12: padded to 16
    (3, 16, 4, 64),    # r = 4 at d = 64: 256-row tiles
]


@pytest.mark.parametrize("shape", BF16_SHAPES, ids=lambda s: "B%d_Hq%d_Hkv%d_d%d" % s)
def test_bf16_small_all_outputs(oracle, shape):
    B, H_q, H_kv, d = shape
    w = inputs.custom(f"bf16_{B}_{H_q}_{H_kv}_{d}", B=B, H_q=H_q, H_kv=H_kv, d=d, L_max=1100,
                      dtype=torch.bfloat16, q_std=0.5, kv_std=1.0, seed=100 + H_q + H_kv + d)
    choices = [1, 7, 8, 9, 127, 128, 129, 255, 256, 257, 1000, 1100]
    lengths = [choices[(i * 5 + H_kv) % len(choices)] for i in range(B)]
    _check(oracle, w, lengths=lengths)


@pytest.mark.parametrize("lengths", [[1], [128], [129], [1100], [1, 1100, 128, 129, 2, 3, 640, 641]])
def test_bf16_length_mix(oracle, lengths):
    w = inputs.custom("bf16_mix", B=len(lengths), H_q=32, H_kv=8, d=128, L_max=1100,
                      dtype=torch.bfloat16, seed=5)
    _check(oracle, w, lengths=lengths)


def test_bf16_many_short_sequences(oracle):
    # more units than CTAs, most of them one partial tile: exercises segment walking
    B = 300
    rng = np.random.default_rng(3)
    lengths = rng.integers(1, 200, size=B).tolist()
    w = inputs.custom("bf16_many", B=B, H_q=16, H_kv=4, d=64, L_max=200, dtype=torch.bfloat16,
                      seed=9)
    _check(oracle, w, lengths=lengths)


@pytest.mark.parametrize("shape", [(2, 8, 2, 64), (3, 16, 16, 128), (2, 32, 1, 128), (1, 128, 1, 64)],
                         ids=lambda s: "B%d_Hq%d_Hkv%d_d%d" % s)
def test_f32_small_all_outputs(oracle, shape):
    B, H_q, H_kv, d = shape
    w = inputs.custom("f32", B=B, H_q=H_q, H_kv=H_kv, d=d, L_max=700, dtype=torch.float32, seed=11)
    lengths = [[1, 63, 64, 65, 700][(i + H_kv) % 5] for i in range(B)]
    _check(oracle, w, lengths=lengths)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_append_bit_exact(dtype):
    w = inputs.custom("app", B=5, H_q=8, H_kv=4, d=128, L_max=50, dtype=dtype, seed=21)
    x = inputs.make_inputs(w, lengths=[1, 2, 50, 17, 30], poison=False)
    out, lens, status, g = run_step(x)
    assert status == 0
    kc = g["k_cache"].cpu()
    vc = g["v_cache"].cpu()
    k0 = x["k_cache"].clone()
    v0 = x["v_cache"].clone()
    for b in range(w.B):
        t = int(x["seq_lens_pre"][b])
        k0[b, t] = x["k_new"][b]
        v0[b, t] = x["v_new"][b]
    assert torch.equal(kc.view(torch.int16 if dtype == torch.bfloat16 else torch.int32),
                       k0.view(torch.int16 if dtype == torch.bfloat16 else torch.int32))
    assert torch.equal(vc.view(torch.int16 if dtype == torch.bfloat16 else torch.int32),
                       v0.view(torch.int16 if dtype == torch.bfloat16 else torch.int32))
    assert torch.equal(lens.cpu(), x["lengths"])


def test_append_overflow_reported_and_skipped():
    w = inputs.custom("ovf", B=3, H_q=8, H_kv=2, d=64, L_max=16, seed=22)
    x = inputs.make_inputs(w, lengths=[16, 5, 16], poison=False)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    lens = torch.tensor([16, 4, 20], dtype=torch.int32, device="cuda")  # 16, 20: no room
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    import grouped_query_attention_decode_b200 as gqa
    gqa.kv_append(g["k_new"], g["v_new"], g["k_cache"], g["v_cache"], lens, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & gqa.STATUS_APPEND_OVERFLOW
    assert lens.cpu().tolist() == [16, 5, 20]
    assert torch.equal(g["k_cache"][0].cpu(), x["k_cache"][0])
    assert torch.equal(g["k_cache"][2].cpu(), x["k_cache"][2])
    assert torch.equal(g["k_cache"][1, 4].cpu(), x["k_new"][1])


def test_empty_and_out_of_range_lengths(oracle):
    import grouped_query_attention_decode_b200 as gqa
    w = inputs.custom("empty", B=4, H_q=16, H_kv=4, d=128, L_max=300, seed=23)
    x = inputs.make_inputs(w, lengths=[0, 300, 0, 77], poison=True)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    lens = torch.tensor([0, 300, 301, 77], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # decode only (no append): rows [0, n) are the attended rows; poison covers [n-1, L_max)
    kc, vc = g["k_cache"].clone(), g["v_cache"].clone()
    kc[1, 299] = g["k_new"][1]
    vc[1, 299] = g["v_new"][1]
    kc[3, 76] = g["k_new"][3]
    vc[3, 76] = g["v_new"][3]
    out = gqa.decode(g["q"], kc, vc, lens, x["scale"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & gqa.STATUS_SEQLEN_RANGE
    o = out.cpu()
    assert torch.equal(o[0], torch.zeros_like(o[0])) and torch.equal(o[2], torch.zeros_like(o[2]))
    xx = dict(x)
    xx["k_cache"], xx["v_cache"] = kc.cpu(), vc.cpu()
    xx["lengths"] = torch.tensor([0, 300, 0, 77], dtype=torch.int32)
    ref = oracle_step(oracle, xx, [1, 3], append=False)
    assert max_err(out, ref) <= TOL[torch.bfloat16]


def test_deterministic():
    w = inputs.custom("det", B=4, H_q=32, H_kv=8, d=128, L_max=2000, seed=24)
    x = inputs.make_inputs(w)
    a, _, _, _ = run_step(x)
    b, _, _, _ = run_step(x)
    assert torch.equal(a, b)


@pytest.mark.parametrize("pattern", ["growing", "jump", "shrinking"])
def test_running_max_paths(oracle, pattern):
    """The running maximum is raised only when a tile's scores exceed it by more than a margin;
    scores that grow along the sequence, jump once by far more than the margin, or start high and
    shrink exercise both the lazy path and the rescaling path."""
    w = inputs.custom("maxpath", B=3, H_q=16, H_kv=2, d=128, L_max=1500, dtype=torch.bfloat16,
                      q_std=0.5, kv_std=1.0, seed=33)
    x = inputs.make_inputs(w, lengths=[1500, 700, 300])
    t = torch.arange(w.L_max, dtype=torch.float32)
    if pattern == "growing":
        f = 1.0 + 6.0 * t / w.L_max
    elif pattern == "jump":
        f = torch.where(t < 600, torch.full_like(t, 0.3), torch.full_like(t, 6.0))
    else:
        f = 6.0 - 5.0 * t / w.L_max
    x["k_cache"] = (x["k_cache"].float() * f[None, :, None, None]).to(torch.bfloat16)
    out, lens, status, _ = run_step(x)
    assert status == 0
    assert torch.isfinite(out).all()
    ref = oracle_step(oracle, x)
    assert max_err(out, ref) <= TOL[torch.bfloat16]

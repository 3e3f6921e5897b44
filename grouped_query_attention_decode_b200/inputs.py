"""Seeded synthetic inputs for one GQA decode step.

This module draws random numbers and lays them out; it does none of the attention arithmetic.
The CUDA path and the CPU oracle are both fed from it, so both see identical bytes.

Recipe (all draws from one ``torch.Generator('cpu')`` seeded with the workload's seed):
  1. q        [B, H_q, d]            ~ N(0, 1) * q_std
  2. k_cache  [B, L_max, H_kv, d]    ~ N(0, 1) * kv_std, drawn one sequence (b) at a time
  3. v_cache  [B, L_max, H_kv, d]    same
  4. k_new    [B, H_kv, d]           ~ N(0, 1) * kv_std
  5. v_new    [B, H_kv, d]           same
  6. lengths  [B]  either the fixed length, or uniform integers in [1, L_max] (ragged)
Each float is drawn in fp32 and rounded to the storage dtype with round-to-nearest-even.
An FP8 (e4m3) cache (``kv_format="e4m3"``) first draws k_scale, v_scale [H_kv] =
kv_std * U(0.75, 1.25) / 32; its cache steps 2-3 draw N(0, 1) * 32 and round it to the nearest
e4m3 code (torch's float8_e4m3fn), so code * scale is again ~ N(0, kv_std^2); q, k_new and v_new
stay in the workload's dtype (bf16) and the append quantises the new rows.
``lengths`` is the number of rows attended AFTER this step's append, so the cache starts with
``seq_lens = lengths - 1`` and the append writes row ``lengths - 1``.  With Q > 1 query tokens
per sequence (speculative verification), q is [B, Q, H_q, d], k_new/v_new are [B, Q, H_kv, d]
and the append writes the last Q rows.  Cache rows at or beyond
``lengths - 1`` hold no data the step may read; ``poison=True`` fills them with NaN so a kernel
that reads them poisons its output.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H_q: int
    H_kv: int
    d: int
    L_max: int
    dtype: torch.dtype
    q_std: float
    kv_std: float
    seed: int
    length: int | None = None          # fixed attended length; None = ragged U{1..L_max}
    scale: float | None = None         # None = 1/sqrt(d)
    window: int = 0                    # > 0: sliding window, attend the last `window` rows
    page_size: int = 0                 # > 0: the cache lives in a paged pool (see make_paged)
    queries: int = 1                   # query tokens per sequence (speculative verification)
    kv_format: str = ""                # "e4m3": FP8 cache codes with per-head scales
    note: str = field(default="", compare=False)

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)

    @property
    def elem_bytes(self) -> int:
        """Bytes of one cached K or V element."""
        if self.kv_format == "e4m3":
            return 1
        return torch.tensor([], dtype=self.dtype).element_size()

    @property
    def fp8(self) -> bool:
        return self.kv_format == "e4m3"


# The pages' workloads, each named by what it is.
WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_fp32", B=1, H_q=8, H_kv=2, d=64, L_max=256, dtype=torch.float32,
                 q_std=1.0, kv_std=1.0, seed=0, length=256, scale=1.0 / 8.0,
                 note="tiny GQA step, group size 4"),
        Workload("llama2_70b_layer", B=16, H_q=64, H_kv=8, d=128, L_max=4096,
                 dtype=torch.bfloat16, q_std=0.5, kv_std=0.5, seed=1, length=4096,
                 note="Llama-2-70B-shaped attention layer, GQA-8"),
        Workload("t5xxl_g64_mha", B=32, H_q=64, H_kv=64, d=64, L_max=2048,
                 dtype=torch.bfloat16, q_std=1.0, kv_std=1.0, seed=2, length=2048,
                 scale=1.0 / 8.0, note="T5-XXL-shaped head sweep, G=64 (MHA)"),
        Workload("t5xxl_g8", B=32, H_q=64, H_kv=8, d=64, L_max=2048,
                 dtype=torch.bfloat16, q_std=1.0, kv_std=1.0, seed=2, length=2048,
                 scale=1.0 / 8.0, note="T5-XXL-shaped head sweep, G=8"),
        Workload("t5xxl_g1_mqa", B=32, H_q=64, H_kv=1, d=64, L_max=2048,
                 dtype=torch.bfloat16, q_std=1.0, kv_std=1.0, seed=2, length=2048,
                 scale=1.0 / 8.0, note="T5-XXL-shaped head sweep, G=1 (MQA)"),
        Workload("mqa_long", B=64, H_q=32, H_kv=1, d=128, L_max=8192, dtype=torch.bfloat16,
                 q_std=0.5, kv_std=1.0, seed=3, length=8192,
                 note="MQA with a long cache"),
        Workload("ragged_long", B=32, H_q=32, H_kv=8, d=128, L_max=32768, dtype=torch.bfloat16,
                 q_std=1.0, kv_std=1.0, seed=4, length=None,
                 note="ragged long-context batch, lengths uniform in [1, 32768]"),
        Workload("llama2_70b_layer_paged16", B=16, H_q=64, H_kv=8, d=128, L_max=4096,
                 dtype=torch.bfloat16, q_std=0.5, kv_std=0.5, seed=1, length=4096, page_size=16,
                 note="the Llama-2-70B-shaped layer in a paged pool of 16-row pages"),
        Workload("llama2_70b_layer_spec4", B=16, H_q=64, H_kv=8, d=128, L_max=4096,
                 dtype=torch.bfloat16, q_std=0.5, kv_std=0.5, seed=1, length=4096, queries=4,
                 note="the Llama-2-70B-shaped layer verifying 4 drafted tokens per sequence"),
        Workload("ragged_long_window4096", B=32, H_q=32, H_kv=8, d=128, L_max=32768,
                 dtype=torch.bfloat16, q_std=1.0, kv_std=1.0, seed=4, length=None, window=4096,
                 note="the ragged batch with a Mistral-style sliding window of 4096 rows"),
        Workload("llama2_70b_layer_fp8", B=16, H_q=64, H_kv=8, d=128, L_max=4096,
                 dtype=torch.bfloat16, q_std=0.5, kv_std=0.5, seed=1, length=4096, kv_format="e4m3",
                 note="the Llama-2-70B-shaped layer with an FP8 (e4m3) cache"),
        Workload("ragged_long_fp8", B=32, H_q=32, H_kv=8, d=128, L_max=32768, dtype=torch.bfloat16,
                 q_std=1.0, kv_std=1.0, seed=4, length=None, kv_format="e4m3",
                 note="the ragged long-context batch with an FP8 (e4m3) cache"),
    ]
}


def custom(name="custom", *, B, H_q, H_kv, d, L_max, dtype=torch.bfloat16, q_std=1.0,
           kv_std=1.0, seed=1234, length=None, scale=None, window=0, page_size=0,
           queries=1, kv_format="") -> Workload:
    return Workload(name, B=B, H_q=H_q, H_kv=H_kv, d=d, L_max=L_max, dtype=dtype, q_std=q_std,
                    kv_std=kv_std, seed=seed, length=length, scale=scale, window=window,
                    page_size=page_size, queries=queries, kv_format=kv_format)


E4M3_NAN = 0x7F


def _e4m3_codes(shape, gen) -> torch.Tensor:
    """uint8 e4m3 codes of N(0, 1) * 32 rounded to nearest (torch's float8_e4m3fn)."""
    x = torch.randn(shape, generator=gen, dtype=torch.float32).mul_(32.0).clamp_(-448.0, 448.0)
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def _normal(shape, gen, std, dtype):
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def make_inputs(w: Workload, lengths=None, poison: bool = False) -> dict:
    """Host (CPU) tensors for one append + decode step of workload ``w``.

    ``lengths`` (a list of B ints in [0, L_max]) overrides the drawn lengths; a length of 0
    means "no append, nothing to attend" for tests of the empty case (seq_lens starts at 0 and
    the caller skips the append).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    Qn = w.queries
    q = _normal((w.B, w.H_q, w.d) if Qn == 1 else (w.B, Qn, w.H_q, w.d), g, w.q_std, w.dtype)
    extra = {}
    if w.fp8:
        u = torch.rand((2, w.H_kv), generator=g, dtype=torch.float32)
        extra["k_scale"] = (w.kv_std * (0.75 + 0.5 * u[0]) / 32.0).float()
        extra["v_scale"] = (w.kv_std * (0.75 + 0.5 * u[1]) / 32.0).float()
        k_cache = torch.empty((w.B, w.L_max, w.H_kv, w.d), dtype=torch.uint8)
        v_cache = torch.empty_like(k_cache)
        for b in range(w.B):
            k_cache[b] = _e4m3_codes((w.L_max, w.H_kv, w.d), g)
        for b in range(w.B):
            v_cache[b] = _e4m3_codes((w.L_max, w.H_kv, w.d), g)
    else:
        k_cache = torch.empty((w.B, w.L_max, w.H_kv, w.d), dtype=w.dtype)
        v_cache = torch.empty_like(k_cache)
        for b in range(w.B):
            k_cache[b] = _normal((w.L_max, w.H_kv, w.d), g, w.kv_std, w.dtype)
        for b in range(w.B):
            v_cache[b] = _normal((w.L_max, w.H_kv, w.d), g, w.kv_std, w.dtype)
    new_shape = (w.B, w.H_kv, w.d) if Qn == 1 else (w.B, Qn, w.H_kv, w.d)
    k_new = _normal(new_shape, g, w.kv_std, w.dtype)
    v_new = _normal(new_shape, g, w.kv_std, w.dtype)
    if w.length is not None:
        drawn = torch.full((w.B,), w.length, dtype=torch.int32)
    else:
        drawn = torch.randint(1, w.L_max + 1, (w.B,), generator=g, dtype=torch.int64).to(torch.int32)
    if lengths is not None:
        drawn = torch.tensor(list(lengths), dtype=torch.int32)
        assert drawn.shape == (w.B,)
    seq_lens_pre = torch.clamp(drawn - Qn, min=0).to(torch.int32)
    if poison:
        nan = E4M3_NAN if w.fp8 else float("nan")
        for b in range(w.B):
            k_cache[b, int(seq_lens_pre[b]):] = nan
            v_cache[b, int(seq_lens_pre[b]):] = nan
    return {
        "q": q, "k_cache": k_cache, "v_cache": v_cache, "k_new": k_new, "v_new": v_new,
        "seq_lens_pre": seq_lens_pre, "lengths": drawn, "scale": w.softmax_scale, **extra,
    }


def make_paged(x: dict, page_size: int, extra_pages: int = 3, seed: int = 99) -> dict:
    """Scatter the contiguous caches of ``x`` ([B, L_max, H_kv, d], L_max a multiple of
    page_size) into a pool of pages in a seeded random order: block_table[b, j] is the pool
    page holding rows [j*page_size, (j+1)*page_size) of sequence b.  ``extra_pages`` unused
    pages (NaN) are mixed in.  Returns {"k_pool", "v_pool", "block_table"}."""
    kc, vc = x["k_cache"], x["v_cache"]
    B, L_max, H_kv, d = kc.shape
    assert L_max % page_size == 0
    max_pages = L_max // page_size
    n_pages = B * max_pages + extra_pages
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    perm = torch.randperm(n_pages, generator=g)[: B * max_pages].to(torch.int32)
    nan = E4M3_NAN if kc.dtype == torch.uint8 else float("nan")  # unused pages hold NaN
    k_pool = torch.full((n_pages, page_size, H_kv, d), nan, dtype=kc.dtype)
    v_pool = torch.full_like(k_pool, nan)
    k_pool[perm.long()] = kc.reshape(B * max_pages, page_size, H_kv, d)
    v_pool[perm.long()] = vc.reshape(B * max_pages, page_size, H_kv, d)
    return {"k_pool": k_pool, "v_pool": v_pool, "block_table": perm.reshape(B, max_pages).contiguous()}


def attended_rows(w: Workload, n: int) -> int:
    """Rows a sequence of length n attends: all of them, or the last `window`."""
    n = int(n)
    return min(n, w.window) if w.window > 0 else n


def ideal_kv_bytes(w: Workload, lengths) -> int:
    """K and V bytes one decode step must read: 2 * sum(attended rows) * H_kv * d * element
    size."""
    return 2 * int(sum(attended_rows(w, n) for n in lengths)) * w.H_kv * w.d * w.elem_bytes

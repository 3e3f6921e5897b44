"""Element, byte and multiply counts of the KV cache and of one decode step.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

- KV-cache size: 2 * B * N * L * H_kv * d_h * bytes, the leading 2 being K and V.
  "从MHA到GQA" (blog.gzher.com), section on why the problem moved from computing attention to
  storing K/V ("KVCache ≈ 2BNLH_kv d_h b"); the same count with H_kv = H in "GQA 阅读笔记",
  section 3 (KV cache), and without the byte factor in the lesson "r-tf2-gqa" (what shrinks).
- Cached elements per token and layer: MHA 2 H_q d_h, GQA 2 G d_h, MQA 2 d_h;
  "从MHA到GQA", section on MLA, the per-structure cache table.
- Multiplies of the attention body: h * n * n * d for the scores and again for the weighted sum
  in a full pass over n positions, with no g in it; "r-tf2-gqa", section on what shrinks.
  For one decode step (one query row per head) the same count is h * n * d per product.
"""


def kv_cache_elements(B: int, N_layers: int, L: int, H_kv: int, d_h: int) -> int:
    return 2 * B * N_layers * L * H_kv * d_h


def kv_cache_bytes(B: int, N_layers: int, L: int, H_kv: int, d_h: int, bytes_per: int) -> int:
    return kv_cache_elements(B, N_layers, L, H_kv, d_h) * bytes_per


def cache_elements_per_token(H_kv: int, d_h: int) -> int:
    """Per token and layer; H_kv = H_q is MHA, H_kv = G is GQA, H_kv = 1 is MQA."""
    return 2 * H_kv * d_h


def attention_multiplies_full_pass(h: int, n: int, d: int) -> dict:
    """Multiplies of one layer's attention body over n positions (no g anywhere)."""
    return {"scores": h * n * n * d, "weighted_sum": h * n * n * d}


def decode_step_multiplies(seq_lens, H_q: int, d: int) -> int:
    """Multiplies of one decode step's attention: each query head dots n_b key rows and
    weights n_b value rows, so 2 * sum(n_b) * H_q * d; independent of H_kv."""
    return 2 * sum(int(n) for n in seq_lens) * H_q * d


def decode_step_kv_elements(seq_lens, H_kv: int, d: int) -> int:
    """Cached K and V elements one decode step has to read: 2 * sum(n_b) * H_kv * d."""
    return 2 * sum(int(n) for n in seq_lens) * H_kv * d

"""Cache-size and multiply counts against the numbers the pages print (tests/golden/)."""
import os

import pytest

from oracle import counts

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name), encoding="utf-8"):
        if line.strip() and not line.startswith("#"):
            rows.append([c.strip() for c in line.split("|")])
    return rows


@pytest.mark.parametrize("row", _rows("kv_cache_sizes.txt"), ids=lambda r: r[0])
def test_printed_kv_cache_sizes(row):
    _, B, N, L, H_kv, d, nbytes, expected, _cite = row
    got = counts.kv_cache_bytes(int(B), int(N), int(L), int(H_kv), int(d), int(nbytes))
    assert got == int(expected)


@pytest.mark.parametrize("row", _rows("cache_elements_per_token.txt"), ids=lambda r: r[0])
def test_printed_elements_per_token(row):
    _, H_kv, d, expected, _cite = row
    assert counts.cache_elements_per_token(int(H_kv), int(d)) == int(expected)


def test_cache_shrinks_with_kv_heads_and_multiplies_do_not():
    # lesson "r-tf2-gqa": the cache is proportional to g, the attention multiplies have no g
    lens = [5, 17, 2048]
    base_elems = counts.decode_step_kv_elements(lens, 64, 128)
    base_mults = counts.decode_step_multiplies(lens, 64, 128)
    for g in (64, 8, 1):
        assert counts.decode_step_kv_elements(lens, g, 128) * 64 == base_elems * g
        assert counts.kv_cache_elements(1, 32, 4096, g, 128) * 64 == counts.kv_cache_elements(1, 32, 4096, 64, 128) * g
        assert counts.decode_step_multiplies(lens, 64, 128) == base_mults
    full = counts.attention_multiplies_full_pass(8, 10, 4)
    assert full == {"scores": 3200, "weighted_sum": 3200}


@pytest.mark.parametrize("row", _rows("kv_bytes_ratios.txt"), ids=lambda r: r[0])
def test_printed_fp8_bandwidth_ratios(row):
    _, h_a, b_a, h_b, b_b, expected, _cite = row
    for B, N, L, d in ((1, 1, 1, 128), (16, 80, 4096, 128), (3, 2, 17, 64)):
        a = counts.kv_cache_bytes(B, N, L, int(h_a), d, int(b_a))
        b = counts.kv_cache_bytes(B, N, L, int(h_b), d, int(b_b))
        assert a == int(expected) * b

"""CPU tests of the measurement helpers in bench.py: the comment-stripped source hash that gates
a profile's DRAM bytes, the percentile of the kernel timings and the number of rotating cache
copies that keeps every step HBM-cold."""
import json
import math

import pytest

import bench


def test_strip_comments_ignores_comments_and_layout_only():
    a = "int f(int x) {  // doubles\n    return 2 * x; /* twice */\n}\n"
    b = "int f(int x) {\n/* a longer\n   comment */ return 2 * x;\n}"
    c = "int f(int x) { return 3 * x; }"
    assert bench.strip_comments(a) == bench.strip_comments(b)
    assert bench.strip_comments(a) != bench.strip_comments(c)


def test_profiled_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    kernel, workload = "split_tc_kernel", "llama2_70b_layer"
    monkeypatch.setattr(bench, "PROFILE_DIR", str(tmp_path))
    path = tmp_path / f"split_tc_{workload}.json"
    # no summary: nothing quoted
    assert bench.profiled_traffic(workload, kernel) is None
    path.write_text(json.dumps({"kernel_source_hash": bench.kernel_source_hash(kernel),
                                "dram_bytes_per_launch_full_size": 123}))
    assert bench.profiled_traffic(workload, kernel) == 123
    # a capture of other code: not quoted
    path.write_text(json.dumps({"kernel_source_hash": "0" * 16, "dram_bytes_per_launch_full_size": 123}))
    assert bench.profiled_traffic(workload, kernel) is None
    # a kernel the bench does not know
    assert bench.profiled_traffic(workload, "other_kernel") is None


def test_committed_profiles_name_their_kernel_sources():
    # every committed summary records the comment-stripped hash it was taken on, and the ones
    # of the current sources are quoted
    import glob
    import os
    for p in glob.glob(os.path.join(bench.PROFILE_DIR, "*.json")):
        d = json.load(open(p))
        assert len(d["kernel_source_hash"]) == 16
        assert d["dram_bytes_per_launch_full_size"] >= d["algorithmic_bytes_per_launch"]


@pytest.mark.parametrize("v,p,want", [
    ([5.0], 10, 5.0),
    ([1.0, 2.0, 3.0, 4.0, 5.0], 50, 3.0),
    ([1.0, 2.0, 3.0, 4.0, 5.0], 10, 1.4),
    ([5.0, 1.0, 4.0, 2.0, 3.0], 90, 4.6),
    ([], 50, None),
])
def test_percentile_interpolates(v, p, want):
    got = bench.percentile(v, p)
    assert (got is None and want is None) or math.isclose(got, want)


@pytest.mark.parametrize("step_mb,want", [(268.4, 2), (2307.1, 2), (16.8, 17), (0.3, 886)])
def test_cache_copies_cover_twice_the_l2(step_mb, want):
    l2 = 132_644_864  # the B200's L2 as the device reports it
    n = bench.cache_copies(l2, int(step_mb * 1e6))
    assert n == want
    # a copy is read again only after >= 2 x L2 of other K/V
    assert (n - 1) * step_mb * 1e6 >= 2 * l2


def test_cache_copies_capped():
    # a step of a few KB would need thousands of copies; the count stops at 1024
    assert bench.cache_copies(132_644_864, 4096) == 1024

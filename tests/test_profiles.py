"""The committed DRAM counters that bench.py's roofline "traffic" reads: well formed, and keyed by
the sha1 of each kernel source together with every file it includes."""
import json
import os
import re
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    sys.path.insert(0, ROOT)
    import bench
    return bench


def test_traffic_file_is_well_formed():
    rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    units = rec["units_per_launch"]
    assert units > 0 and rec["command"].startswith("python bench.py")
    for name, k in rec["kernels"].items():
        assert os.path.exists(os.path.join(ROOT, k["source"])), name
        assert re.fullmatch(r"[0-9a-f]{40}", k["sources_sha1"]), name
        assert abs(k["bytes_per_unit"] - (k["dram_read_mb"] + k["dram_write_mb"]) * 1e6 / units) < 0.01, name
        # counters at or near the algorithmic bytes: no kernel re-reads its inputs
        assert 0.8 * k["algorithmic_bytes_per_unit"] < k["bytes_per_unit"] < 1.2 * k["algorithmic_bytes_per_unit"]


def test_source_closure_follows_includes():
    bench = _bench()
    files = bench.source_closure("kv_cache_vector_compress_b200/csrc/tq_compress_tc.cu")
    assert "kv_cache_vector_compress_b200/csrc/tq_compress_tc.cu" in files
    assert "kv_cache_vector_compress_b200/csrc/tq_sm100.cuh" in files
    assert "include/tq.h" in files  # reached through tq_internal.cuh
    # the hash changes with any included file's contents (names and bytes both enter it)
    h = bench.sources_sha1("kv_cache_vector_compress_b200/csrc/tq_compress_tc.cu")
    assert re.fullmatch(r"[0-9a-f]{40}", h)
    assert h != bench.sources_sha1("kv_cache_vector_compress_b200/csrc/tq_attend_planes.cu")

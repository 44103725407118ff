"""bench.py reports roofline.traffic only while the kernels' code matches the
hash recorded with the ncu capture: comment edits keep the hash, code edits
change it."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_code_only_ignores_comments_not_code():
    import bench
    a = "int f(int x) {\n  // one\n  return x + 1;  /* two */\n}\n"
    b = "int f(int x) {\n  // a longer comment\n\n  return x + 1;\n  /* block\n     over lines */\n}\n"
    c = "int f(int x) {\n  return x + 2;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_recorded_traffic_is_reported_only_for_matching_code():
    import json
    import bench
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))["gemv_scalar"]
    got = bench.profiled_traffic("gemv_scalar")
    if rec["source_sha"] == bench.kernel_source_hash():
        assert got == rec["dram_bytes_per_launch"]
    else:  # kernels changed since the capture: no traffic figure
        assert got is None

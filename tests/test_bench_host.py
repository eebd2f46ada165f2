"""Host-side logic of bench.py that needs no GPU."""
import os
import sys

sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))
import bench  # noqa: E402


def test_traffic_key_ignores_comments_but_not_code():
    """The DRAM-traffic record is keyed to the code of the sources that decide
    the GEMM launch mix: editing a comment keeps the key, editing code (even a
    constant) changes it, so a stale capture is reported as null."""
    src = "int f(int a) {  // scale\n  /* block\n comment */ return 2 * a;\n}\n"
    same = "int f(int a) {   // a different comment\n\n  return 2 * a;   \n}\n"
    other = "int f(int a) {\n  return 3 * a;\n}\n"
    key = lambda text: bench.traffic_source_sha(lambda name: text)
    assert key(src) == key(same)
    assert key(src) != key(other)


def test_traffic_record_matches_the_tree():
    """The committed record was taken on code identical to the working tree's
    (the bench would report it as null otherwise)."""
    import json
    with open(os.path.join(bench.ROOT, "profiles", "gemm_traffic.json")) as f:
        d = json.load(f)
    assert d["source_sha256"] == bench.traffic_source_sha()
    assert d["bytes_per_launch"] > 0

"""Host-side logic of bench.py (no GPU): the hash that decides whether a
recorded DRAM-traffic figure still belongs to the kernel sources, and the
recorded figures' own consistency."""
import json
import os

import bench


def test_code_hash_ignores_comments_and_whitespace():
    a = 'int f(int x) {\n    return x + 1;  // one more\n}\n/* block */ const char *s = "//kept";\n'
    b = 'int f(int x) { return x + 1; }\nconst char *s = "//kept";\n'
    c = 'int f(int x) { return x + 2; }\nconst char *s = "//kept";\n'
    d = 'int f(int x) { return x + 1; }\nconst char *s = "//changed";\n'
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(b) != bench._code_only(c)
    assert bench._code_only(b) != bench._code_only(d)  # string literals are code
    assert bench._code_only("char q = '\\'';  // quote") == "char q = '\\'';"


def test_src_hash_reads_every_kernel_source():
    seen = []

    def read(name):
        seen.append(name)
        return "x"
    h1 = bench.src_hash(read)
    assert seen == list(bench.KERNEL_SOURCES)
    assert h1 != bench.src_hash(lambda name: "y")
    for name in bench.KERNEL_SOURCES:
        assert os.path.exists(os.path.join(bench.CSRC, name)), name


def test_recorded_traffic_entries_are_consistent():
    path = os.path.join(bench.ROOT, "profiles", "dram_traffic.json")
    with open(path) as f:
        rec = json.load(f)
    for name, e in rec.items():
        assert e["dram_bytes_per_launch"] == e["dram_read_bytes"] + e["dram_write_bytes"] or \
            abs(e["dram_bytes_per_launch"] - e["dram_read_bytes"] - e["dram_write_bytes"]) <= 2, name
        assert "--clock-control none" in e["command"], name
        assert len(e["src_sha"]) == 16, name

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
        assert set(e.get("sources") or bench.KERNEL_SOURCES) <= set(bench.KERNEL_SOURCES), name
        if name.endswith("_bwd"):   # the gradient kernels: every source but the host pipeline
            assert tuple(e["sources"]) == bench.GRAD_SOURCES, name
        else:
            assert tuple(e["sources"]) == bench.FORWARD_SOURCES, name


def test_forward_sources_leave_out_only_the_gradient_and_host_pipeline_sources():
    assert set(bench.KERNEL_SOURCES) - set(bench.FORWARD_SOURCES) == \
        set(bench.GRAD_ONLY_SOURCES) | set(bench.HOST_ONLY_SOURCES)
    assert set(bench.KERNEL_SOURCES) - set(bench.GRAD_SOURCES) == set(bench.HOST_ONLY_SOURCES)
    # no device source pulls in a gradient header or the host pipeline
    for name in bench.FORWARD_SOURCES:
        if name == "capi.cu":   # the library's entry points, all of them
            continue
        with open(os.path.join(bench.CSRC, name), encoding="utf-8") as f:
            text = f.read()
        for g in bench.GRAD_ONLY_SOURCES + bench.HOST_ONLY_SOURCES:
            assert f'#include "{g}"' not in text, (name, g)
    # the host pipeline defines no kernel
    with open(os.path.join(bench.CSRC, "capi_host.cuh"), encoding="utf-8") as f:
        assert "__global__" not in f.read()


def test_recorded_traffic_is_keyed_to_the_entry_sources(tmp_path, monkeypatch):
    fwd = bench.src_hash(names=bench.FORWARD_SOURCES)
    rec = {"a": {"src_sha": fwd, "sources": list(bench.FORWARD_SOURCES), "dram_bytes_per_launch": 7},
           "b": {"src_sha": fwd, "dram_bytes_per_launch": 8},        # no list: every source
           "c": {"src_sha": fwd, "sources": ["nope.cu"], "dram_bytes_per_launch": 9}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("a") == 7
    assert bench.recorded_traffic("b") is None
    assert bench.recorded_traffic("c") is None
    assert bench.recorded_traffic("missing") is None

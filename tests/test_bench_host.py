"""Host logic of bench.py that needs no GPU: the code hash that decides
whether a recorded DRAM traffic figure still describes the kernels."""
import json
import os

import bench


def test_code_hash_ignores_comments_and_layout():
    a = 'int f(int x) {\n  return x + 1;  // add one\n}\n/* trailing\n   block */\n'
    b = '/* a new header comment */\nint f(int x)\n{\n    return x + 1;\n}\n'
    assert bench._code_only(a) == bench._code_only(b)


def test_code_hash_sees_code_and_string_literals():
    base = bench._code_only('asm("add.f32 %0, %1, %2;" : "=f"(r));  // x')
    assert bench._code_only('asm("sub.f32 %0, %1, %2;" : "=f"(r));') != base
    # comment markers inside a string literal are code, not comments
    s = bench._code_only('const char *u = "http://host/*x*/"; int y;')
    assert "http://host/*x*/" in s and "int y;" in s
    assert bench._code_only("char c = '\\''; int z; // done") == "char c = '\\''; int z;"


def test_recorded_traffic_matches_current_kernels():
    # Every record names kernel sources that exist; a record whose code hash
    # no longer matches is reported as unknown (None) by the bench, never as
    # a stale number.
    d = json.load(open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")))
    for key, rec in d.items():
        if key.startswith("_"):
            continue
        got = bench.load_traffic(key)
        if bench.source_hash(*rec["sources"]) == rec["source_hash"]:
            assert got == rec["bytes_per_launch"]
        else:
            assert got is None
    assert bench.load_traffic("no-such-kernel") is None

"""Host logic of bench.py that needs no GPU: the code hash that decides
whether a recorded DRAM traffic figure still describes the kernels, and the
reference arm (the fp64 oracle on the host cores) and its JSON line."""
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


def test_reference_arm_line():
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints
    one JSON line with the contract's keys, on the GPU arm's workload and
    metric."""
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=bench.ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == "prefill tokens/s" and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 1 and d["warmup"] >= 3 and d["n_gpus"] == 1
    assert d["config"]["workload"].startswith("elu_bf16_fwd")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["unit"] == d["unit"]
    assert cb["cores"] >= 1 and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0

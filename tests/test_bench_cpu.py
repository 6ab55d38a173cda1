"""Host-side pieces of bench.py that need no GPU."""
import json

import bench


def test_code_digest_ignores_comments_and_whitespace(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "a.cu").write_text('int f(int x) { return x + 1; }  // one\n/* two */\n')
    base = bench.code_digest(["a.cu"])
    (tmp_path / "a.cu").write_text('// header\nint f(int x)\n{\n    return x + 1;  /* other */\n}\n')
    assert bench.code_digest(["a.cu"]) == base
    (tmp_path / "a.cu").write_text('int f(int x) { return x + 2; }\n')
    assert bench.code_digest(["a.cu"]) != base
    # a comment marker inside a string literal is code
    (tmp_path / "a.cu").write_text('const char* s = "// not a comment"; int f(int x) { return x + 1; }\n')
    with_str = bench.code_digest(["a.cu"])
    (tmp_path / "a.cu").write_text('const char* s = ""; int f(int x) { return x + 1; }\n')
    assert bench.code_digest(["a.cu"]) != with_str


def test_recorded_traffic_follows_the_code(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cu").write_text("int k() { return 1; }\n")
    rec = {"w": {"sources": ["k.cu"], "code_digest": bench.code_digest(["k.cu"]),
                 "traffic_bytes": 123}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("w") == 123
    (tmp_path / "k.cu").write_text("int k() { return 1; }  // comment only\n")
    assert bench.recorded_traffic("w") == 123
    (tmp_path / "k.cu").write_text("int k() { return 2; }\n")
    assert bench.recorded_traffic("w") is None
    assert bench.recorded_traffic("other") is None

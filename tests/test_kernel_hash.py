"""bench.kernel_hash: the profiles in profiles/ are keyed by a hash of the
kernel's code; commentary and blank space do not change it, code does (a
profile taken on other code is then not reported as the bench's traffic)."""
import bench


def test_kernel_hash_ignores_comments_not_code(tmp_path):
    a = tmp_path / "a.cuh"
    b = tmp_path / "b.cuh"
    c = tmp_path / "c.cuh"
    a.write_text("// header\nint f(int x) { return x + 1; }  // add one\n/* block\n note */\n")
    b.write_text("int f(int x)   {\n  return x + 1;\n}\n// another note\n")
    c.write_text("int f(int x) { return x + 2; }\n")
    assert bench.kernel_hash([str(a)]) == bench.kernel_hash([str(b)])
    assert bench.kernel_hash([str(a)]) != bench.kernel_hash([str(c)])



def test_traffic_is_reported_only_for_the_code_it_was_taken_on(tmp_path, monkeypatch):
    import json
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"w": {"kernel_hash": "aaaa", "dram_bytes_per_launch": 123}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_hash", lambda sources=None: "aaaa")
    assert bench.load_traffic("w") == 123
    assert bench.load_traffic("other") is None
    monkeypatch.setattr(bench, "kernel_hash", lambda sources=None: "bbbb")
    assert bench.load_traffic("w") is None

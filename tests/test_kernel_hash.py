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


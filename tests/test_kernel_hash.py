"""bench.kernel_hash: the profiles in profiles/ are keyed by a hash of the
kernel's code; commentary and blank space do not change it, code does."""
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


def test_profiles_are_keyed_by_the_current_kernel():
    # the committed traffic figures belong to the kernel as it is
    assert bench.load_traffic("tinyllama-ctx0") is not None
    assert bench.load_traffic("llama7b-ctx2048") is not None

"""bench.py's kernel-source digest, which decides whether a committed DRAM
traffic figure still belongs to the kernel being timed: line comments and
blank lines do not change it, code does."""
import bench


def _digest(tmp_path, text):
    (tmp_path / "k.cu").write_text(text)
    old = bench.ROOT
    bench.ROOT = str(tmp_path)
    try:
        return bench.source_digest(["k.cu"])
    finally:
        bench.ROOT = old


def test_comments_and_blank_lines_do_not_count(tmp_path):
    a = _digest(tmp_path, "int f(int x) {\n  return x + 1;\n}\n")
    b = _digest(tmp_path, "// f adds one\nint f(int x) {  // trailing note\n\n  return x + 1;\n}\n")
    assert a == b


def test_code_changes_count(tmp_path):
    a = _digest(tmp_path, "int f(int x) {\n  return x + 1;\n}\n")
    b = _digest(tmp_path, "int f(int x) {\n  return x + 2;\n}\n")
    assert a != b


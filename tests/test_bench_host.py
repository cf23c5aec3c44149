"""Host logic of bench.py that needs no GPU: the kernel-source hash that keys
the recorded DRAM traffic follows the code and not its comments."""

import os
import shutil

import bench


def test_code_only_strips_comments_and_keeps_literals():
    src = ('int a = 1;  // trailing\n/* block\n   comment */ const char* s = "not // a comment";\n'
           "\n  char c = '/'; x = y / z; /* end */\n")
    out = bench._code_only(src)
    assert "trailing" not in out and "block" not in out and "end" not in out
    assert '"not // a comment"' in out and "'/'" in out and "x = y / z;" in out
    assert "\n\n" not in out


def test_kernel_hash_ignores_comments_and_follows_code(tmp_path):
    csrc = os.path.join(bench.ROOT, "rwkv_wkv_linear_b200", "csrc")
    copy = tmp_path / "csrc"
    shutil.copytree(csrc, copy)
    base = bench.kernel_source_hash(str(copy))
    assert base == bench.kernel_source_hash()
    f = copy / "wkv4_scan.cuh"
    text = f.read_text()
    f.write_text("// a new comment line\n" + text.replace("namespace wkv4 {", "namespace wkv4 {  /* c */", 1))
    assert bench.kernel_source_hash(str(copy)) == base
    f.write_text(text + "\nstatic const int unused_constant = 1;\n")
    assert bench.kernel_source_hash(str(copy)) != base


def test_kernel_hash_leaves_out_the_host_pipeline(tmp_path):
    """wkv4_host.cpp only chains the forward's calls: a change there keeps the
    recorded kernel traffic valid; a change to the launchers does not."""
    csrc = os.path.join(bench.ROOT, "rwkv_wkv_linear_b200", "csrc")
    copy = tmp_path / "csrc"
    shutil.copytree(csrc, copy)
    base = bench.kernel_source_hash(str(copy))
    f = copy / "wkv4_host.cpp"
    f.write_text(f.read_text() + "\nstatic const int another_constant = 2;\n")
    assert bench.kernel_source_hash(str(copy)) == base
    g = copy / "wkv4_api.cpp"
    g.write_text(g.read_text() + "\nstatic const int another_constant = 2;\n")
    assert bench.kernel_source_hash(str(copy)) != base

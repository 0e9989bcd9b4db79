"""bench.py's DRAM-traffic records (CPU).

The bench line's roofline carries the DRAM bytes of one launch of the
dominant kernel, read from profiles/dram_traffic.txt, and only while the
record was taken on the kernel's current source: a record names the source
by a hash of its code with comments and blank lines removed. Checked:
- editing a comment keeps the hash, editing code changes it;
- every workload's attention and o_proj records match the current sources
  (a kernel changed without re-taking its records fails here, rather than
  printing a roofline with no traffic).
"""
import os

import pytest

import bench
from mla_causal_attention_attn_b200 import inputs


def _write(root, name, text):
    d = os.path.join(root, "mla_causal_attention_attn_b200", "csrc")
    os.makedirs(d, exist_ok=True)
    with open(os.path.join(d, name), "w") as f:
        f.write(text)


def test_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = "// header\nint f(int x) {\n  return x + 1;  // one\n}\n"
    _write(tmp_path, "k.cu", base)
    h0 = bench.kernel_source_sha("k.cu")
    _write(tmp_path, "k.cu", "/* other\n header */\n\nint f(int x) {\n  return x + 1;\n}\n\n")
    assert bench.kernel_source_sha("k.cu") == h0
    _write(tmp_path, "k.cu", "// header\nint f(int x) {\n  return x + 2;  // one\n}\n")
    assert bench.kernel_source_sha("k.cu") != h0


def test_recorded_traffic_needs_the_current_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    _write(tmp_path, "k.cu", "int f() { return 1; }\n")
    sha = bench.kernel_source_sha("k.cu")
    os.makedirs(tmp_path / "profiles")
    (tmp_path / "profiles" / "dram_traffic.txt").write_text(
        "# comment\n"
        f"k.cu wl_a {sha} 1234\n"
        "k.cu wl_b 0000000000000000 99\n")
    assert bench.recorded_traffic("k.cu", "wl_a") == 1234.0
    assert bench.recorded_traffic("k.cu", "wl_b") is None   # taken on another source
    assert bench.recorded_traffic("k.cu", "wl_c") is None   # never taken


@pytest.mark.parametrize("kernel_file", ["attn_prefill.cu", "oproj_gemm.cu"])
@pytest.mark.parametrize("workload", sorted(inputs.WORKLOADS))
def test_committed_records_match_current_sources(kernel_file, workload):
    assert bench.recorded_traffic(kernel_file, workload) is not None, (
        f"profiles/dram_traffic.txt has no record of {kernel_file} at {workload} "
        f"for its current source ({bench.kernel_source_sha(kernel_file)})")

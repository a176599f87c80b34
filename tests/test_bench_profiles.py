"""bench.py's link between the committed ncu traffic summaries and the source they were taken
on (CPU): the hash covers the code of the GEMM sources with comments and whitespace removed, so a
comment edit keeps a summary valid and a code edit makes the bench report traffic as null."""
import os
import sys

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, REPO)

import bench  # noqa: E402


def _write(root, name, text):
    with open(os.path.join(root, name), "w", encoding="utf-8") as f:
        f.write(text)


def test_hash_ignores_comments_and_whitespace_but_not_code(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "REPO", str(tmp_path))
    _write(tmp_path, "k.cu", "// kernel\nint f(int a) {\n    return a + 1;   /* one */\n}\n")
    h0 = bench.source_sha(["k.cu"])
    _write(tmp_path, "k.cu", "// the kernel, reworded\nint f(int a) {\n  return a + 1; /* one,\n two */\n}\n")
    assert bench.source_sha(["k.cu"]) == h0
    _write(tmp_path, "k.cu", "// kernel\nint f(int a) {\n    return a + 2;   /* one */\n}\n")
    assert bench.source_sha(["k.cu"]) != h0


def test_traffic_read_only_for_the_current_code(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "REPO", str(tmp_path))
    os.makedirs(tmp_path / "profiles")
    src = ["a.cu", "b.cuh"]
    monkeypatch.setattr(bench, "GEMM_SOURCES", src)
    _write(tmp_path, "a.cu", "int g() { return 3; }\n")
    _write(tmp_path, "b.cuh", "#pragma once\n")
    sha = bench.source_sha(src)
    _write(tmp_path / "profiles", "expert_gateup_decode_traffic.txt",
           f"kernel: expert_gateup\ndram_bytes_per_launch: 5100750592\nsource_sha: {sha}\n")
    assert bench.profiled_traffic("expert_gateup", "decode") == 5100750592.0
    assert bench.profiled_traffic("expert_down", "decode") is None          # no summary
    _write(tmp_path, "a.cu", "int g() { return 4; }\n")                       # the kernel changed
    assert bench.profiled_traffic("expert_gateup", "decode") is None


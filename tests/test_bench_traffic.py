"""bench.py's recorded DRAM traffic: the ncu byte counts in profiles/traffic.json
are reported only while the kernel sources match the code they were taken on.
The match is on the code with comments and blank lines left out, so that a
comment edit keeps the figure and a code edit drops it (the tests work on a
copy of the sources and of the capture file)."""

import json
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_only_drops_comments_and_blank_lines():
    src = "int a; // note\n\n/* block\n comment */ int b;\n   \nint c;  // trailing\n"
    assert bench._code_only(src) == "int a;\n int b;\nint c;"


def test_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    base = "__global__ void k(int* p) {\n  p[0] = 1;\n}\n"
    (tmp_path / "a.cu").write_text(base)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.source_hash(["a.cu"])
    (tmp_path / "a.cu").write_text("// header\n" + base.replace("p[0] = 1;", "p[0] = 1;  // store"))
    assert bench.source_hash(["a.cu"]) == h0
    (tmp_path / "a.cu").write_text(base.replace("p[0] = 1;", "p[0] = 2;"))
    assert bench.source_hash(["a.cu"]) != h0


def test_recorded_traffic_follows_the_source_hash():
    """A capture whose hash matches the current kernel code is reported
    (scaled by algorithmic bytes for another launch size); one that does not
    is dropped."""
    with open(bench.TRAFFIC_FILE) as f:
        rec = json.load(f)
    for kernel in ("attention", "pack_tma"):
        got = bench.recorded_traffic(kernel)
        if rec[kernel]["source_hash"] != bench.source_hash(bench.KERNEL_SOURCES[kernel]):
            assert got is None, kernel
            continue
        assert got == rec[kernel]["bytes_per_launch"]
        half = bench.recorded_traffic(kernel, rec[kernel]["algorithmic_bytes"] / 2)
        assert abs(half - got / 2) <= 1e-6 * got


def test_recorded_traffic_dropped_after_a_code_change(tmp_path, monkeypatch):
    for kernel in ("attention",):
        for rel in bench.KERNEL_SOURCES[kernel]:
            dst = tmp_path / rel
            dst.parent.mkdir(parents=True, exist_ok=True)
            shutil.copy(os.path.join(ROOT, rel), dst)
    shutil.copytree(os.path.join(ROOT, "profiles"), tmp_path / "profiles")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "profiles" / "traffic.json"))
    with open(bench.TRAFFIC_FILE) as f:
        rec = json.load(f)
    rec["attention"]["source_hash"] = bench.source_hash(bench.KERNEL_SOURCES["attention"])
    with open(bench.TRAFFIC_FILE, "w") as f:
        json.dump(rec, f)
    assert bench.recorded_traffic("attention") is not None
    src = tmp_path / bench.KERNEL_SOURCES["attention"][0]
    src.write_text(src.read_text() + "\n// a comment only\n")
    assert bench.recorded_traffic("attention") is not None
    src.write_text(src.read_text() + "\nstatic int unused_code_change = 0;\n")
    assert bench.recorded_traffic("attention") is None

"""Host-side logic of bench.py: the source fingerprint that keeps a recorded ncu DRAM-traffic
figure valid, and the lookup that drops the figure once the kernel's code has changed."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

KERNEL = """// a kernel
__global__ void k(float *x) {
    /* scale
       in place */
    x[threadIdx.x] *= 2.f;   // twice
}
"""


def _write(root, name, text):
    with open(os.path.join(root, name), "w", encoding="utf-8") as f:
        f.write(text)


def test_source_hash_ignores_comments_and_layout(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    _write(tmp_path, "k.cu", KERNEL)
    h0 = bench.source_hash(["k.cu"])
    _write(tmp_path, "k.cu", KERNEL.replace("// twice", "// doubled, with a longer note\n// on two lines")
           .replace("/* scale\n       in place */", "/* scale in place */"))
    assert bench.source_hash(["k.cu"]) == h0
    _write(tmp_path, "k.cu", KERNEL.replace("    x[threadIdx.x]", "\n\n        x[threadIdx.x]"))
    assert bench.source_hash(["k.cu"]) == h0


def test_source_hash_changes_with_the_code(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    _write(tmp_path, "k.cu", KERNEL)
    h0 = bench.source_hash(["k.cu"])
    _write(tmp_path, "k.cu", KERNEL.replace("2.f", "3.f"))
    assert bench.source_hash(["k.cu"]) != h0
    _write(tmp_path, "k.cu", KERNEL.replace("*= 2.f", "+= 2.f"))
    assert bench.source_hash(["k.cu"]) != h0


def test_traffic_figure_is_dropped_once_the_code_changes(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    os.makedirs(tmp_path / "profiles")
    _write(tmp_path, "k.cu", KERNEL)
    rec = {"wl/B1": {"kern": {"bytes_per_launch": 123.0, "sources": ["k.cu"],
                              "source_hash": bench.source_hash(["k.cu"])}}}
    _write(tmp_path / "profiles", "traffic.json", json.dumps(rec))
    assert bench.ncu_traffic("kern", "wl/B1") == 123.0
    assert bench.ncu_traffic("kern", "other/B1") is None
    _write(tmp_path, "k.cu", KERNEL + "// a comment only\n")
    assert bench.ncu_traffic("kern", "wl/B1") == 123.0
    _write(tmp_path, "k.cu", KERNEL.replace("2.f", "4.f"))
    assert bench.ncu_traffic("kern", "wl/B1") is None


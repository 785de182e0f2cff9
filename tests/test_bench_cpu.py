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



def test_both_arms_report_the_same_config():
    """The reference arm (the oracle) and our arm build the line's config from the same function, for
    the default workload and the others, so the driver sees the same config on both lines."""
    import argparse
    from distilled_ssm_decode_b200 import workloads as W
    w = W.WORKLOADS[bench.DEFAULT_WORKLOAD]
    assert bench.DEFAULT_WORKLOAD == "gen1p3b_bf16" and w.layers == 24
    cfg = bench.line_config(w, w.layers)
    assert cfg["layers"] == 24 and cfg["B"] == 64 and cfg["L"] == 512 and cfg["Dch"] == 2048
    assert "24 independent layers" in cfg["workload"]
    for name, wl in W.WORKLOADS.items():
        assert bench.line_config(wl, wl.layers) == bench.line_config(wl, wl.layers)
    src = open(os.path.join(ROOT, "bench.py")).read()
    # both arms print config=line_config(w, nl) and nothing else under "config"
    assert src.count('"config": line_config(w, nl)') == 2


def test_algorithmic_bytes_match_the_documented_figures():
    from distilled_ssm_decode_b200 import workloads as W
    pre, dec = bench.algorithmic_bytes(W.WORKLOADS["mid_bf16"])
    assert pre == 269_484_032 and dec == 2_162_688
    pre, dec = bench.algorithmic_bytes(W.WORKLOADS["gen1p3b_bf16"])
    assert pre * 24 == 13_287_555_072 and dec * 24 == 830_472_192
    pre, _ = bench.algorithmic_bytes(W.WORKLOADS["long_prefill_bf16"])
    assert pre == 402_751_488
    _, dec = bench.algorithmic_bytes(W.WORKLOADS["decode_sweep_bf16"].with_(B=1024))
    assert dec == 1_107_296_256

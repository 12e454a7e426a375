"""The bench line's `traffic` comes from a committed ncu summary only while
the kernel's code is the code that was captured: the source hash ignores
comments and layout, and any change of code drops the counters."""
import json

import bench

SRC = """// a kernel
__global__ void k(int *p) {
    /* block
       comment */
    p[0] = 1;   // trailing
}
"""


def _tree(tmp_path, text):
    d = tmp_path / "int8_weight_only_b200" / "csrc"
    d.mkdir(parents=True, exist_ok=True)
    (d / "k.cuh").write_text(text)


def test_hash_ignores_comments_and_layout(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    _tree(tmp_path, SRC)
    h0 = bench.kernel_source_hash(["k.cuh"])
    _tree(tmp_path, SRC.replace("// a kernel", "// the kernel, reworded").replace("    p[0]", "\n        p[0]"))
    assert bench.kernel_source_hash(["k.cuh"]) == h0
    _tree(tmp_path, SRC.replace("p[0] = 1;", "p[0] = 2;"))
    assert bench.kernel_source_hash(["k.cuh"]) != h0


def test_traffic_only_while_the_code_matches(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    _tree(tmp_path, SRC)
    (tmp_path / "profiles").mkdir()
    entry = {"k": {"bytes_per_launch": 123456, "source_hash": bench.kernel_source_hash(["k.cuh"])}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(entry))
    assert bench.measured_traffic("k", ["k.cuh"]) == 123456.0
    _tree(tmp_path, SRC.replace("p[0] = 1;", "p[1] = 1;"))
    assert bench.measured_traffic("k", ["k.cuh"]) is None
    assert bench.measured_traffic("absent", ["k.cuh"]) is None


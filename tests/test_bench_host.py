"""Host logic of bench.py that needs no GPU: the per-workload layout choice
and the lookup of committed DRAM-traffic figures (taken only when the kernel
code -- comments aside -- and, for the forward, the layout are those the
figure was measured on)."""
import json

import bench


def test_auto_layout_covers_every_bench_workload():
    assert set(bench.AUTO_LAYOUT) == {1, 2, 3, 4}
    assert set(bench.AUTO_LAYOUT.values()) <= {"corners", "quads", "padded", "linear"}


def _entry(tmp_path, monkeypatch, layout="corners", digest=None):
    (tmp_path / "k.cu").write_text("int f(int x) { return x + 1; }  // add one\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d = bench.code_digest(["k.cu"]) if digest is None else digest
    table = {"forward_kernel": {"w": {"sources": ["k.cu"], "code_sha256_16": d,
                                      "dram_bytes_per_launch": 123, "layout": layout}}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(table))


def test_traffic_is_taken_for_the_same_source_and_layout(tmp_path, monkeypatch):
    _entry(tmp_path, monkeypatch)
    assert bench.traffic_for("forward_kernel", "w", "corners") == 123


def test_traffic_is_null_for_another_layout_or_workload(tmp_path, monkeypatch):
    _entry(tmp_path, monkeypatch)
    assert bench.traffic_for("forward_kernel", "w", "quads") is None
    assert bench.traffic_for("forward_kernel", "other workload", "corners") is None
    assert bench.traffic_for("adjoint_kernel", "w", "corners") is None


def test_traffic_is_null_once_the_code_changed(tmp_path, monkeypatch):
    _entry(tmp_path, monkeypatch, digest="0" * 16)
    assert bench.traffic_for("forward_kernel", "w", "corners") is None
    _entry_dir = tmp_path / "second"
    _entry_dir.mkdir()
    _entry(_entry_dir, monkeypatch)
    (_entry_dir / "k.cu").write_text("int f(int x) { return x + 2; }\n")
    assert bench.traffic_for("forward_kernel", "w", "corners") is None


def test_a_comment_edit_keeps_the_traffic(tmp_path, monkeypatch):
    _entry(tmp_path, monkeypatch)
    (tmp_path / "k.cu").write_text("// adds one\nint f(int x)\n{\n    return x + 1;  /* one */\n}\n")
    assert bench.traffic_for("forward_kernel", "w", "corners") == 123


def test_committed_traffic_names_the_bench_workloads():
    with open(bench.os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    names = {bench.config_block(bench.workload(c), c)["workload"] for c in (2, 3)}
    for kernel in ("forward_kernel", "adjoint_kernel"):
        assert set(table[kernel]) <= names
        for entry in table[kernel].values():
            assert entry["dram_bytes_per_launch"] > 0
    for entry in table["forward_kernel"].values():
        assert entry["layout"] in ("corners", "quads")

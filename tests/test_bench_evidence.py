"""bench.py reports a kernel's committed DRAM traffic figure only while the
kernel's device sources are the ones that were profiled: the source hash
ignores comments and blank lines, and any code change turns the figure off."""
import importlib.util
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_code_only_ignores_comments_and_blank_lines():
    b = _bench()
    a = "int x = 1;  // one\n\n/* block\n comment */int y;\n"
    c = "int x = 1;\n// another comment\nint y;   \n"
    assert b._code_only(a) == b._code_only(c) == "int x = 1;\nint y;"
    assert b._code_only("int x = 2;") != b._code_only("int x = 1;")


def test_committed_traffic_figures_are_used_only_for_the_profiled_kernels():
    b = _bench()
    for kind, srcs in (("fwd", b.KERNEL_SOURCES), ("bwd", b.BWD_KERNEL_SOURCES)):
        d = json.load(open(os.path.join(ROOT, "profiles", f"attn_{kind}_c3_traffic.json")))
        current = d["kernel_src_sha256"] == b.kernel_source_hash(srcs)
        assert b.load_traffic("c3", kind) == (d["dram_bytes_per_launch"] if current else None)


def test_traffic_figure_is_dropped_when_the_hash_differs(tmp_path, monkeypatch):
    b = _bench()
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "attn_fwd_c3_traffic.json").write_text(
        json.dumps({"kernel_src_sha256": "0" * 16, "dram_bytes_per_launch": 1.0}))
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    monkeypatch.setattr(b, "kernel_source_hash", lambda sources=None: "f" * 16)
    assert b.load_traffic("c3", "fwd") is None
    (prof / "attn_fwd_c3_traffic.json").write_text(
        json.dumps({"kernel_src_sha256": "f" * 16, "dram_bytes_per_launch": 1.0}))
    assert b.load_traffic("c3", "fwd") == 1.0

"""The DRAM-traffic table of bench.py is keyed by a hash of kernel code, not of comments (CPU only)."""
import importlib.util
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_traffic_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_code_only_drops_comments_and_keeps_strings():
    b = _load_bench()
    src = 'int a; // one\n/* two\n three */ int b;\n\n   \nasm("ld.shared [%0]; // not a comment");\n'
    assert b.code_only(src) == 'int a;\n int b;\nasm("ld.shared [%0]; // not a comment");'
    assert b.code_only('s = "a \\" // b"; // c') == 's = "a \\" // b";'


def test_comment_edits_keep_the_hash_and_code_edits_change_it(tmp_path, monkeypatch):
    b = _load_bench()
    csrc = tmp_path / "nvfp4_weight_only_route_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("gemv.cu", "mma.cu", "common.cuh", "internal.h"):
        (csrc / f).write_text("// header\nint f() { return 1; }\n")
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    h0 = b.kernel_source_hash("gemv_gate_up")
    (csrc / "gemv.cu").write_text("// another header\n\nint f() { return 1; }  // same code\n")
    assert b.kernel_source_hash("gemv_gate_up") == h0
    (csrc / "gemv.cu").write_text("int f() { return 2; }\n")
    assert b.kernel_source_hash("gemv_gate_up") != h0
    assert b.kernel_source_hash("mma_gate_up") != b.kernel_source_hash("gemv_gate_up")


def test_table_entries_are_well_formed_and_only_used_when_the_code_matches():
    """An entry is read only while its hash names the current code; otherwise the bench line
    reports traffic as null (a kernel changed since the capture)."""
    b = _load_bench()
    table = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
    for workload, stages in table.items():
        if workload.startswith("_"):
            continue
        for stage, ent in stages.items():
            h = ent["kernel_source_hash"]
            assert len(h) == 16 and int(h, 16) >= 0
            assert ent["dram_bytes_per_launch"] > 0
            expect = ent["dram_bytes_per_launch"] if h == b.kernel_source_hash(stage) else None
            assert b.ncu_traffic(workload, stage) == expect

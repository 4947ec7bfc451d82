"""Host-side bookkeeping of bench.py (no GPU): the source fingerprint that ties
the stored DRAM counters to the kernel code ignores comments and layout but not
code, and a changed kernel reports no traffic."""

import importlib.util
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def test_code_of_drops_comments_keeps_code_and_strings():
    b = load_bench()
    src = 'int a = 1; // one\n/* block\n comment */ asm("mov %0, 1; // kept");\n\n  int  b;'
    assert b.code_of(src) == 'int a = 1; asm("mov %0, 1; // kept"); int b;'
    assert b.code_of(src) == b.code_of(src.replace("// one", "// changed comment"))
    assert b.code_of(src) != b.code_of(src.replace("a = 1", "a = 2"))


def test_changed_kernel_reports_no_traffic(monkeypatch):
    b = load_bench()
    cfg = b.W.CONFIGS["dsv3"]
    pt = b.padded_total_of(cfg)
    fam = "gemm_fprop_up"
    _, group, sha = b.TRAFFIC_CAPTURE["families"][fam]
    monkeypatch.setattr(b, "source_hash", lambda g: sha)
    t = b.measured_traffic(fam, cfg, pt)
    assert t is not None and t > 0
    monkeypatch.setattr(b, "source_hash", lambda g: "0" * 12)
    assert b.measured_traffic(fam, cfg, pt) is None


def test_traffic_scales_with_algorithmic_bytes(monkeypatch):
    b = load_bench()
    monkeypatch.setattr(b, "source_hash", lambda g: dict(
        (grp, sha) for _, grp, sha in b.TRAFFIC_CAPTURE["families"].values())[g])
    cap = b.W.CONFIGS[b.TRAFFIC_CAPTURE["config"]]
    for fam, (bytes_cap, _, _) in b.TRAFFIC_CAPTURE["families"].items():
        t = b.measured_traffic(fam, cap, b.padded_total_of(cap))
        assert abs(t - bytes_cap) <= 1e-6 * bytes_cap, fam

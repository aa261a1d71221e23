"""Host-side logic of the benchmark (no GPU): workload names, the removal of
planted overflow steps from the timed loops, and the rule that stored ncu
traffic figures are used only for the device code they were taken on."""
import json

import bench
import workloads as W
from loss_scaled_fp32_b200 import build as mbuild


def test_workload_names_and_shifted_variant():
    cfg, shift = bench.workload_of("ragged20k_shift2B")
    assert cfg.name == "ragged20k" and shift
    cfg, shift = bench.workload_of("gpt_1p3b")
    assert cfg.name == "gpt_1p3b" and not shift
    for name in bench.DEFAULT_EXTRA.split(","):
        bench.workload_of(name)                     # every default entry resolves


def test_timed_loops_draw_no_planted_overflow():
    flat = W.get("flat1m")
    assert flat.injections(5)                       # the workload plants +inf at step 5
    stripped = bench.without_injections(flat)
    assert all(stripped.injections(s) == [] for s in range(1, 11))
    assert stripped.sizes == flat.sizes and stripped.scale0 == flat.scale0
    assert flat.injections(5)                       # the original is untouched


def test_traffic_figures_only_for_the_current_kernels(tmp_path, monkeypatch):
    path = tmp_path / "dram_traffic.json"
    rec = {"update_kernel": {"dram_bytes_per_param": 20.5, "capture": "test capture",
                             "kernel_source_sha256": mbuild.kernel_digest()},
           "check_kernel": {"dram_bytes_per_param": 2.0, "capture": "old capture",
                            "kernel_source_sha256": "0" * 64}}
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    traffic, source = bench.load_traffic("update_kernel", 1000)
    assert traffic == 20500.0 and "test capture" in source
    traffic, source = bench.load_traffic("check_kernel", 1000)
    assert traffic is None and "predate" in source
    traffic, source = bench.load_traffic("refresh_kernel", 1000)
    assert traffic is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.json"))
    assert bench.load_traffic("update_kernel", 1000)[0] is None


def test_l2_note_flags_resident_state():
    assert "L2-resident" in bench.l2_note(1 << 20)
    assert "larger than L2" in bench.l2_note(354_823_168)


def test_kernel_digest_ignores_comments_and_layout_only():
    """The digest that ties stored ncu figures to the device code changes
    with the code, not with its comments or line breaks."""
    from loss_scaled_fp32_b200 import build as mbuild
    a = "int f(int x)\n{\n    return x + 1;  // one more\n}\n"
    b = "/* a note */ int f(int x) { return x + 1; }"
    c = "int f(int x)\n{\n    return x + 2;  // one more\n}\n"
    assert mbuild._code_only(a) == mbuild._code_only(b)
    assert mbuild._code_only(a) != mbuild._code_only(c)
    assert len(mbuild.kernel_digest()) == 64

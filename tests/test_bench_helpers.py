"""Host-side helpers of bench.py: the recorded ncu traffic is reported only
while the attention kernel's code matches the code that was profiled."""
import os
import re

import bench


def test_strip_comments_keeps_code_and_strings():
    src = 'int a; // one\n/* two */ const char* s = "x // y /* z */"; int b; /* three\n four */ int c;'
    out = bench.strip_comments(src)
    assert "one" not in out and "two" not in out and "three" not in out and "four" not in out
    assert '"x // y /* z */"' in out
    assert "int a;" in out and "int b;" in out and "int c;" in out


def test_recorded_traffic_follows_the_kernel_code(tmp_path, monkeypatch):
    # a profile summary recorded against the current kernel code
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "attn_fwd_kernel_full_s4096_ncu.md").write_text(
        "traffic_bytes_per_launch: 4.2e7\nkernel_source_sha256: %s\n" % bench.kernel_code_sha256())
    assert bench.recorded_traffic("full_s4096", str(prof)) == 4.2e7
    # no profile for other workloads
    assert bench.recorded_traffic("sliding_s1024", str(prof)) is None
    # a code edit (not a comment) invalidates it: hash a modified copy
    copies = []
    for src in bench.KERNEL_SOURCES:
        dst = tmp_path / os.path.basename(src)
        text = open(src).read()
        dst.write_text(text)
        copies.append(str(dst))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", copies)
    assert bench.recorded_traffic("full_s4096", str(prof)) is not None
    with open(copies[0], "a") as f:
        f.write("\n// a comment changes nothing\n")
    assert bench.recorded_traffic("full_s4096", str(prof)) is not None
    with open(copies[0], "a") as f:
        f.write("\nstatic int extra_code = 1;\n")
    assert bench.recorded_traffic("full_s4096", str(prof)) is None


def test_profile_records_traffic_and_hash():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    text = open(os.path.join(root, "profiles", "attn_fwd_kernel_full_s4096_ncu.md")).read()
    assert re.search(r"traffic_bytes_per_launch: \d+", text)
    assert re.search(r"kernel_source_sha256: [0-9a-f]{64}", text)


def test_backward_flops_are_five_contractions_per_pair_and_head():
    import workloads as W
    w = W.make("sliding_s1024")
    # forward: 2 contractions (QK^T, PV) x 2 FLOPs x 128 x 32 heads per pair
    assert w.flops() == 2 * 2 * 128 * 32 * w.valid_pairs()
    assert bench.bwd_flops(w) == 5 * 2 * 128 * 32 * w.valid_pairs()


def test_backward_cpu_baseline_reports_one_thread_and_its_sample():
    import workloads as W
    r = bench.bwd_cpu_baseline(W.make("sliding_s1024"), budget_s=0.05)
    assert r["kind"] == "oracle" and r["cores"] == 1 and r["unit"] == bench.UNIT
    assert r["value"] > 0 and "first" in r["sample"] and "sliding_s1024" in r["sample"]


def test_backward_workloads_are_selectable():
    import workloads as W
    for name in W.CONFIGS:
        assert (bench.BWD_PREFIX + name)[len(bench.BWD_PREFIX):] == name


def test_soak_loads_for_its_duration_and_skips_under_profile():
    class A:
        pass
    a = A()
    a.profile, a.soak = True, 5.0
    calls = []
    bench.soak(a, lambda: calls.append(1), lambda: None)
    assert calls == []                      # profiler runs take no soak
    a.profile, a.soak = False, 0.05
    syncs = []
    bench.soak(a, lambda: calls.append(1), lambda: syncs.append(1))
    assert len(calls) >= 20 and len(calls) % 20 == 0   # whole groups of 20 steps
    assert len(syncs) == len(calls) // 20

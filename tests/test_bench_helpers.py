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
    # the committed profile matches the committed kernel
    assert bench.recorded_traffic("full_s4096") is not None
    # no profile for other workloads
    assert bench.recorded_traffic("sliding_s1024") is None
    # a code edit (not a comment) invalidates it: hash a modified copy
    copies = []
    for src in bench.KERNEL_SOURCES:
        dst = tmp_path / os.path.basename(src)
        text = open(src).read()
        dst.write_text(text)
        copies.append(str(dst))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", copies)
    assert bench.recorded_traffic("full_s4096") is not None
    with open(copies[0], "a") as f:
        f.write("\n// a comment changes nothing\n")
    assert bench.recorded_traffic("full_s4096") is not None
    with open(copies[0], "a") as f:
        f.write("\nstatic int extra_code = 1;\n")
    assert bench.recorded_traffic("full_s4096") is None


def test_profile_records_traffic_and_hash():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    text = open(os.path.join(root, "profiles", "attn_fwd_kernel_full_s4096_ncu.md")).read()
    assert re.search(r"traffic_bytes_per_launch: \d+", text)
    assert re.search(r"kernel_source_sha256: [0-9a-f]{64}", text)

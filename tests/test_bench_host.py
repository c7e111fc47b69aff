"""Host-side pieces of bench.py that need no GPU: the reference arm's refusal
for workloads without a host step, and the source hash that keys the
committed DRAM-traffic captures (comments and blank lines do not count)."""
import contextlib
import io
import json
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_arm_prints_unavailable_without_a_host_step():
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(types.SimpleNamespace(workload="prefill", steps=1, warmup=0), 1, 0)
    line = json.loads(out.getvalue())
    assert line["impl"] == "reference" and "unavailable" in line


def test_code_only_ignores_comments_and_blank_lines():
    a = 'int x = 1;  // note\n\n// whole line\nconst char *s = "a//b";\n'
    b = 'int x = 1;\nconst char *s = "a//b";   // other note\n'
    assert bench._code_only(a) == bench._code_only(b)
    assert '"a//b"' in bench._code_only(a)            # // inside a string is code
    assert bench._code_only("int y = 2;") != bench._code_only("int y = 3;")


def test_every_traffic_record_names_a_kernel_with_sources():
    with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
        rec = json.load(f)
    for key, ent in rec.items():
        kernel = key.split("@")[0]
        assert kernel in bench.KERNEL_SOURCES, key
        assert ent["bytes_per_launch"] > 0 and len(ent["source_hash"]) == 16, key

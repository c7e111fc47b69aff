"""Host-side pieces of bench.py that need no GPU: the reference arm's refusal
for workloads without a host step, the source hash that keys the committed
DRAM-traffic captures (comments and blank lines do not count), the parsing
of the clock samples, and the algorithmic bytes behind the roofline."""
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


def test_clock_summary_parses_samples_and_reasons():
    cs = bench.ClockSampler(0)
    cs.out = "\n".join([
        "1965, 1965, 812.4, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "1950, 1965, 990.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "1965, 1965, 1001.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "[N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",   # unreadable
        "short line",
    ])
    s = cs.summary()
    assert s == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "samples": 3, "reasons": ["sw_power_cap"]}
    cs.out = "1400, 1965, 700, 0x8, Not Active, Active, Not Active, Not Active"
    assert cs.summary()["reasons"] == ["hw_thermal_slowdown"]
    cs.out = ""
    assert cs.summary() is None


def test_roofline_bytes_follow_the_oracle_footprint():
    # the decode GEMV's algorithmic bytes are the packed layer (the oracle's
    # footprint, pinned to the pages' scorecard) minus U, which the tail reads
    sys.path.insert(0, ROOT)
    from oracle import dvssq_oracle as O
    for M, K, r in ((2560, 10240, 16), (10240, 2560, 24), (512, 2048, 32), (8192, 2048, 24)):
        n_sal = K // 8
        assert bench.packed_bytes(M, K, r, n_sal) == O.packed_bytes(M, K, r, n_sal)
        assert (bench.kernel_bytes("dec_row", M, K, r, n_sal, 1)
                + bench.kernel_bytes("dec_tail", M, K, r, n_sal, 1)) == O.packed_bytes(M, K, r, n_sal)
        assert bench.kernel_bytes("dec_main", M, K, r, n_sal, 16) == bench.kernel_bytes(
            "dec_row", M, K, r, n_sal, 1)
    # encode: W read once in BF16, the codes written once
    M, K = 2560, 10240
    assert bench.kernel_bytes("enc_pass1", M, K, 0, K // 8, 0) == M * K * 2
    assert bench.kernel_bytes("enc_pass2", M, K, 16, K // 8, 0) == (
        M * K * 2 + O.packed_bytes(M, K, 0, K // 8))


def test_reference_arm_line_keeps_the_contract():
    # the oracle arm on the decode workload runs on the host cores (about 10 s)
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(types.SimpleNamespace(workload="decode", steps=1, warmup=0), 1, 0)
    line = json.loads(out.getvalue().strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["unit"] == "GB/s" and line["n_gpus"] == 1
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["config"]["workload"].startswith("spark_down")

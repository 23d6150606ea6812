"""The reference arm of bench.py (the CPU oracle timed on host cores) runs
without a GPU and prints one JSON line with the keys the bench contract
names, for a single timed step and the minimum warm-up."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e")


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [x for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in KEYS:
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["higher_is_better"] is True
    assert d["unit"] == "TFLOP/s" and d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("v3")


def test_warmup_below_three_is_refused():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                          "--warmup", "2"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode != 0 and "warmup" in out.stderr


def test_profiled_traffic_is_keyed_to_code_not_comments():
    # the committed ncu summaries name the attend kernel's code by a hash of
    # its sources without comments: a comment edit keeps the counters valid,
    # a code edit drops them (traffic: null) until the kernel is profiled again
    sys.path.insert(0, ROOT)
    import bench
    assert bench.code_only("int a; // note\n/* block\n comment */ int b;  \n\n  \nint c;") == \
        "int a;\n int b;\nint c;"
    assert bench.code_only("x = 1;\n") != bench.code_only("x = 2;\n")
    h = bench.kernel_hash()
    assert len(h) == 16 and int(h, 16) >= 0

"""bench.py's output contract on CPU: the reference arm (the CPU oracle) prints
one JSON line with the contract's keys, warm-up below three steps is refused,
and the roofline's DRAM traffic is read from the committed profile only while
the profiled kernel source is unchanged."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, timeout=600):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_contract_line():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_warmup_below_three_is_refused():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "2", timeout=120)
    assert r.returncode != 0
    assert "warmup" in (r.stderr + r.stdout)


def test_traffic_only_for_the_profiled_source():
    import hashlib
    import re

    sys.path.insert(0, ROOT)
    import bench

    prof = open(os.path.join(ROOT, "profiles", "q8_gemv_decode_step.md")).read()
    recorded = re.search(r"kernel_source_sha1:\s*([0-9a-f]{40})", prof).group(1)
    src = os.path.join(ROOT, "decode_gemv_qmm_b200", "csrc", "q8_gemv.cu")
    current = hashlib.sha1(open(src, "rb").read()).hexdigest()
    t = bench.committed_traffic("q8_gemv.cu", "q8_gemv_decode_step.md")
    if current == recorded:
        assert isinstance(t, int) and t > 0
    else:  # the kernel changed since the capture: no traffic figure
        assert t is None
    # the step profile was not taken of prefill.cu: its hash never matches
    assert bench.committed_traffic("prefill.cu", "q8_gemv_decode_step.md") is None

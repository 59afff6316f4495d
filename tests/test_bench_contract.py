"""bench.py's output contract on CPU: the reference arm (the fp64 oracle on the host cores) prints
one JSON line with the keys and types the benchmark driver reads, and bad timing arguments are
refused.  The CUDA arm has the same line and runs in the GPU suite's environment only."""
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
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for key, typ in (("metric", str), ("value", float), ("unit", str), ("n_gpus", int),
                     ("steps", int), ("warmup", int), ("ms_per_step", float),
                     ("higher_is_better", bool), ("scaling", str), ("dtype", str), ("data", str),
                     ("config", dict), ("cpu_baseline", dict), ("e2e", dict)):
        assert isinstance(d[key], typ), (key, d.get(key))
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["config"]["workload"] == "ragged_qwen_b128"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_too_few_warmup_steps_are_refused():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "2", timeout=120)
    assert r.returncode != 0
    assert "warmup" in r.stderr


def test_algorithmic_bytes_by_hand():
    # each byte once: a verified row reads D and T and writes its gradient (6V), an unverified
    # row's gradient is zero-filled (2V), a bonus row reads T (2V); plus the per-sequence outputs
    sys.path.insert(0, ROOT)
    import bench
    import numpy as np
    V, k, kt = 10, 4, 5
    # sequence 0: b_k = 1 -> 1 x 60 + 3 x 20 + bonus 20 = 140; sequence 1: b_k = 4 -> 240 + 20 = 260
    outputs = 2 * 4 * (3 + k + 1 + k)
    assert bench.algorithmic_bytes(np.array([1, 4]), k, kt, V) == 140 + 260 + outputs
    # kt = k: no bonus row when b_k = k
    assert bench.algorithmic_bytes(np.array([4]), k, k, V) == 240 + 4 * (3 + k + 1 + k)

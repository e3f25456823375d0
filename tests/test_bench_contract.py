"""bench.py's output contract, on CPU: the reference arm (the oracle) prints one JSON line with
every key the benchmark contract names, a non-zero rank under torchrun prints nothing and exits
0, and --help lists the ops."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BENCH = os.path.join(ROOT, "bench.py")


def _run(args, env=None):
    e = dict(os.environ)
    for key in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        e.pop(key, None)
    e.update(env or {})
    return subprocess.run([sys.executable, BENCH, *args], capture_output=True, text=True,
                          timeout=300, env=e, cwd=ROOT)


def test_reference_arm_line_has_the_contract_keys():
    r = _run(["--impl", "reference", "--workload", "tiny_T128_E16_k2_H256_softmax", "--steps", "2",
              "--warmup", "1"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e", "gpu_launches"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 2
    assert line["higher_is_better"] is True and line["n_gpus"] == 1
    assert line["config"]["workload"] == "tiny_T128_E16_k2_H256_softmax"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    sysinfo = line["system"]
    assert sysinfo["nproc"] >= 1 and "cpu_model" in sysinfo and sysinfo["gpu_name"] is None


def test_reference_arm_other_ranks_exit_quietly():
    r = _run(["--impl", "reference", "--workload", "tiny_T128_E16_k2_H256_softmax", "--steps", "1",
              "--warmup", "1"], env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_help_lists_the_ops():
    r = _run(["--help"])
    assert r.returncode == 0
    for op in ("step", "backward", "stats", "ep"):
        assert op in r.stdout

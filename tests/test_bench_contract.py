"""bench.py's output contract on the CPU: the reference arm (the fp64 oracle timed on the host
cores) prints exactly one JSON line with the keys the benchmark contract asks for, and a rank
other than 0 exits 0 without work or output."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_ref(env_extra):
    env = dict(os.environ, KDN_REF_TOKENS="128", **env_extra)
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_contract_line():
    p = run_ref({})
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 1 and line["warmup"] == 3
    assert line["higher_is_better"] is True and line["unit"] == "tokens/s"
    assert line["config"]["workload"] == "prefill_B4_H16_T4096_d128_bf16"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    p = run_ref({"RANK": "1", "WORLD_SIZE": "2"})
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""


def test_prefill_roofline_numerator_matches_the_documented_bytes():
    """The prefill roofline's algorithmic bytes: per token and head q, k, alpha, sigma (4 x 256 B),
    v and o (2 x 256 B) and r (2 B), plus the final S and P of every (sequence, head), for
    B4 H16 T4096 d128 bf16: 262144 x 1538 + 64 x (128 x 128 + 128) x 4 = 407,404,544 bytes."""
    sys.path.insert(0, ROOT)
    import bench
    w = bench.workload("prefill")
    assert bench.algorithmic_bytes(w) == 262144 * 1538 + 64 * (128 * 128 + 128) * 4 == 407404544

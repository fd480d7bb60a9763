"""The JSON line of bench.py's reference arm (the CPU oracle timed on the host
cores), checked key by key on the tiny workload: the keys every bench line
carries, plus the reference arm's own (impl, cpu_baseline, e2e with no
host-device bytes)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_reference(*extra):
    env = dict(os.environ)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", *extra],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


def test_reference_line_has_every_key():
    line = run_reference("--steps", "2", "--warmup", "1")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["steps"] == 2 and line["warmup"] == 1 and line["n_gpus"] == 1
    assert line["higher_is_better"] is True and line["scaling"] == "weak" and line["data"] == "synthetic"
    assert line["unit"] == "tokens/s" and line["value"] > 0
    cb = line["cpu_baseline"]
    # the value is the sampled tokens per step over the time of a step
    n = int(cb["sample"].split()[0])
    assert abs(line["value"] * line["ms_per_step"] / 1e3 - n) <= 1e-6 * n
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    cfg = line["config"]
    assert cfg["workload"] == "tiny" and cfg["parallelism"] == "single GPU"


def test_every_extra_workload_is_defined_and_small_batches_are_flushed():
    """The workloads the GPU line carries under "workloads" exist, and each
    batch of at most 64 tokens (whose weights can fit in L2) is one that the
    bench times with L2 flushed before every step."""
    sys.path.insert(0, ROOT)
    import bench
    import workloads as wl
    assert bench.DEFAULT_WORKLOAD not in bench.EXTRA_WORKLOADS
    for name in bench.EXTRA_WORKLOADS:
        assert name in wl.WORKLOADS, name
    small = [n for n in bench.EXTRA_WORKLOADS if wl.WORKLOADS[n].T <= 64]
    assert {"skew_t1", "skew_t8", "skew_t64", "tie_t64"} <= set(small)

"""bench.py's reference arm (the CPU oracle) runs without a GPU and prints one
JSON line with the contract's keys; under torchrun only rank 0 prints."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None, args=()):
    env = dict(os.environ, **(extra_env or {}))
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "1", *args],
                         capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    return [l for l in out.stdout.splitlines() if l.strip()]


def test_reference_arm_json_line():
    lines = _run(args=("--workload", "tiny"))
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["config"]["workload"] == "tiny"


def test_reference_arm_other_ranks_print_nothing():
    assert _run({"RANK": "1", "WORLD_SIZE": "2"}, args=("--workload", "tiny")) == []


def test_reference_arm_lowrank_line():
    lines = _run(args=("--workload", "lowrank"))
    d = json.loads(lines[-1])
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["config"]["rank"] == 32 and d["config"]["iters"] == 2 and "bits" not in d["config"]
    assert d["cpu_baseline"]["cores"] >= 1


def test_reference_arm_config_equals_the_gpu_arm_config():
    """With no flags both arms run the default workload (the CogVideoX-like
    one, the largest) and print the same `config` dict."""
    lines = _run(args=("--steps", "1", "--warmup", "0"))
    d = json.loads(lines[-1])
    sys.path.insert(0, ROOT)
    import bench
    argv = sys.argv
    try:
        sys.argv = ["bench.py"]
        args = bench.parse()
    finally:
        sys.argv = argv
    assert args.workload == "cogvideox"
    wl = bench.W.WORKLOADS[args.workload]
    assert d["config"] == bench.quant_config(args, wl, 1)
    assert d["config"]["tokens"] == 17550 and d["config"]["channels"] == 1920
    assert d["config"]["buffers"] == 60 and d["config"]["bits"] == 2

"""bench.py's launch logic on the CPU: `--gpus N` without a torchrun
environment starts N ranks itself and exactly one JSON line comes out (rank
0's), carrying n_gpus = N; a --gpus that disagrees with WORLD_SIZE fails
loudly.  The reference arm (the oracle on the host cores) keeps this
GPU-free."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env["CUDA_VISIBLE_DEVICES"] = ""
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, env=env,
                          capture_output=True, text=True, timeout=600)


def test_gpus_2_without_torchrun_starts_two_ranks_and_prints_one_line():
    r = _run(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
              "--ref-tokens", "4"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2


def test_gpus_disagreeing_with_world_size_fails_loudly():
    r = _run(["--impl", "reference", "--gpus", "4", "--steps", "1", "--warmup", "0"],
             {"WORLD_SIZE": "2", "RANK": "0"})
    assert r.returncode != 0
    assert "WORLD_SIZE" in (r.stderr + r.stdout)

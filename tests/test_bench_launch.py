"""bench.py --gpus N starts N ranks by itself (no GPU: the launch self-test
runs the same relaunch through torch.distributed.run with gloo ranks) and
prints one JSON line from rank 0; a --gpus that disagrees with the torchrun
world size is refused."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _json_lines(text):
    return [json.loads(l) for l in text.splitlines() if l.strip().startswith("{")]


def _env():
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "LOCAL_RANK", "WORLD_SIZE", "MASTER_ADDR", "MASTER_PORT")}
    env["CUDA_VISIBLE_DEVICES"] = ""
    return env


def test_gpus_2_starts_two_ranks():
    out = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--launch-selftest"], cwd=ROOT,
                         capture_output=True, text=True, timeout=300, env=_env())
    assert out.returncode == 0, out.stderr[-3000:]
    lines = _json_lines(out.stdout)
    assert len(lines) == 1, out.stdout
    d = lines[0]
    assert d["n_gpus"] == 2 and sorted(d["ranks"]) == [0, 1] and d["max_over_ranks"] == 2.0


def test_gpus_must_match_world_size():
    env = dict(_env(), WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--launch-selftest"], cwd=ROOT,
                         capture_output=True, text=True, timeout=120, env=env)
    assert out.returncode != 0 and "WORLD_SIZE" in out.stderr
    assert not _json_lines(out.stdout)

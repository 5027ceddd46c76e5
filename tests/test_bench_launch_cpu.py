"""bench.py --gpus N starts N ranks by itself (CPU, gloo): the launch path
the driver's scaling run depends on, with the GPU work left out (--dry-run).
Each rank must run with its own workload seed, and rank 0 must report the
world size it ran with."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _env():
    env = dict(os.environ)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT", "LOCAL_WORLD_SIZE"):
        env.pop(k, None)
    env["CUDA_VISIBLE_DEVICES"] = ""
    return env


def _json_lines(text):
    out = []
    for ln in text.splitlines():
        ln = ln.strip()
        if ln.startswith("{"):
            out.append(json.loads(ln))
    return out


def test_gpus_two_starts_two_ranks_with_their_own_seeds():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run", "--backend",
                        "gloo", "--steps", "5", "--warmup", "3"], cwd=ROOT, env=_env(), capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1, r.stdout                      # rank 0 alone prints
    line = lines[0]
    assert line["dry_run"] is True and line["n_gpus"] == 2 and line["steps"] == 5
    ranks = sorted(line["ranks"], key=lambda x: x["rank"])
    assert [x["rank"] for x in ranks] == [0, 1]
    assert ranks[0]["seed"] != ranks[1]["seed"]           # each rank its own data
    assert ranks[0]["pid"] != ranks[1]["pid"]             # one process per rank


def test_gpus_must_match_the_launcher():
    env = _env()
    env.update(WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "3", "--dry-run", "--backend",
                        "gloo"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "--gpus 3" in r.stderr


def test_single_rank_dry_run():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "1", "--dry-run", "--backend",
                        "gloo", "--steps", "3", "--warmup", "3"], cwd=ROOT, env=_env(), capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-3000:]
    (line,) = _json_lines(r.stdout)
    assert line["n_gpus"] == 1 and len(line["ranks"]) == 1

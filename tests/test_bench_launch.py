"""bench.py's multi-rank launcher on CPU: `--gpus 2` without a launcher environment starts
two ranks under torch.distributed.run (here: the reference arm, whose ranks join a gloo
group and whose rank 0 alone times the oracle), and the printed line reports both the rank
count and the communicator's size.  A launcher that started a different number of ranks
than --gpus asks for is refused."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _env():
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR",
                                                             "MASTER_PORT")}
    env["CUDA_VISIBLE_DEVICES"] = ""
    return env


def test_gpus_two_spawns_two_gloo_ranks_and_reports_them():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, env=_env(), timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout            # rank 0 alone prints
    d = lines[0]
    assert d["impl"] == "reference" and d["n_gpus"] == 2
    assert d["comm"] == {"backend": "gloo", "world_size": 2}
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_world_size_must_match_gpus():
    env = _env()
    env.update(WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--workload", "tiny", "--steps", "1"],
                       capture_output=True, text=True, env=env, timeout=300, cwd=ROOT)
    assert r.returncode != 0
    assert "WORLD_SIZE=1" in r.stderr

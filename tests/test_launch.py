"""CPU: bench.py --gpus N starts its own ranks (one process per GPU) when no
launcher did, and refuses to run on fewer devices than asked for."""
import importlib.util
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_spawn_ranks_starts_two_gloo_ranks(tmp_path):
    bench = _bench()
    probe = os.path.join(ROOT, "tests", "rank_probe.py")
    rc = bench.spawn_ranks(2, probe, [str(tmp_path)], timeout_s=240)
    assert rc == 0
    seen = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert sorted(s["rank"] for s in seen) == [0, 1]
    assert all(s["world"] == 2 and s["rank_sum"] == 1.0 for s in seen)
    assert sorted(s["local_rank"] for s in seen) == [0, 1]


def test_gpus_beyond_the_visible_devices_fail_loudly():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode != 0
    assert "CUDA device" in r.stderr
    assert r.stdout.strip() == ""


def test_world_size_must_match_gpus():
    env = dict(os.environ, WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 2
    assert "WORLD_SIZE=3" in r.stderr

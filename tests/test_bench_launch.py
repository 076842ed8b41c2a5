"""`bench.py --gpus N` starts its own ranks: without a launcher's environment it re-runs itself under
torch.distributed.run, one rank per GPU, and rank 0 prints the one JSON line with the slowest rank's time.

Here the step is the CPU stand-in (`--stub`, gloo), so the launch, the barriers and the max over ranks run
without a GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_spawns_two_ranks_and_both_report():
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR",
                                                              "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--stub", "--steps", "2",
                        "--warmup", "3"], capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["stub"] is True and d["steps"] == 2
    assert len(d["rank_ms"]) == 2 and all(t > 0 for t in d["rank_ms"])
    assert abs(d["ms_per_step"] - max(d["rank_ms"]) / 2) < 1e-9 * d["ms_per_step"] + 1e-12
    assert d["value"] == 2 * 2 / (max(d["rank_ms"]) / 1e3)


def test_single_rank_stub_runs_in_process():
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--stub", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    d = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][0])
    assert d["n_gpus"] == 1 and len(d["rank_ms"]) == 1


def _bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_recorded_line_is_consistent():
    """A line recorded from a B200 run: the decode launch time times the step's decode launches stays within the
    step's time, frac is achieved / peak, achieved is bytes / launch time, ms_per_step is the slowest rank's."""
    b = _bench_module()
    with open(os.path.join(ROOT, "profiles", "bench_line_qwen3_4b_32k.json")) as f:
        line = json.load(f)
    assert b.check_line(line) == []
    rf = line["roofline"]
    assert rf["launch_ms"] * rf["launches_per_step"] <= line["ms_per_step"]
    assert rf["launches_per_step"] == b.T_BLK * b.LAYERS


def test_check_line_flags_a_launch_time_beyond_the_step():
    b = _bench_module()
    with open(os.path.join(ROOT, "profiles", "bench_line_qwen3_4b_32k.json")) as f:
        line = json.load(f)
    line["roofline"]["launch_ms"] = 1.01 * line["ms_per_step"] / line["roofline"]["launches_per_step"]
    assert any("exceeds ms_per_step" in m for m in b.check_line(line))

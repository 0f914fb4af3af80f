"""bench.py's reference arm (the fp64 oracle timed on the host) keeps the JSON
line contract, on the tiny workload; ranks other than 0 print nothing.  CPU only."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
        "cpu_baseline", "e2e")


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "tiny_T64_H1_d16_fp32", "--steps", "2", "--warmup", "3"],
                          capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)


def test_reference_arm_json_line():
    r = _run({})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    for k in KEYS:
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["steps"] == 2 and line["warmup"] == 3 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "tiny_T64_H1_d16_fp32"
    assert isinstance(line["config"]["seed"], int)   # the input draw's seed travels with the line


def test_reference_arm_other_ranks_silent():
    r = _run({"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_warmup_below_three_rejected():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--warmup", "2"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode != 0


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    bench.barrier(world)
    # per-rank step times; every rank must report the slowest
    got = bench.max_over_ranks([3.0, 7.5, 5.25][rank], world)
    bench.barrier(world)
    dist.destroy_process_group()
    with open(os.path.join(out, f"rank{rank}.json"), "w") as f:
        json.dump(got, f)


def test_max_over_ranks_under_gloo(tmp_path):
    """The bench's cross-rank reduction (max of the per-rank step times, which
    sets value = all ranks' tokens / slowest time) with 2 and 3 gloo ranks on
    the CPU."""
    import socket
    import torch.multiprocessing as mp
    for world in (2, 3):
        with socket.socket() as s:
            s.bind(("127.0.0.1", 0))
            port = s.getsockname()[1]
        out = tmp_path / f"w{world}"
        out.mkdir()
        mp.start_processes(_rank_main, args=(world, port, str(out)), nprocs=world, join=True,
                           start_method="spawn")
        want = max([3.0, 7.5, 5.25][:world])
        for r in range(world):
            assert json.load(open(out / f"rank{r}.json")) == want

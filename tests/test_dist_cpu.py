"""The benchmark's multi-rank plumbing on CPU (gloo, world size 2): process-group set-up from the
torchrun environment, whole-job aggregation (units summed, time maxed over ranks), the barrier, and
the reference arm run as two ranks where rank 0 alone works and prints."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench

    r, w = bench.dist_init("gloo")
    units, seconds = 100.0 * (rank + 1), 0.5 + rank
    total, tmax, value = bench.aggregate(units, seconds)
    bench.barrier()
    mx = bench.reduce_scalar(float(rank), "max")
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"rank": r, "world": w, "total": total, "tmax": tmax, "value": value, "max_rank": mx}, f)
    dist.destroy_process_group()


def test_aggregate_over_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    for rank in range(2):
        got = json.load(open(tmp_path / f"rank{rank}.json"))
        assert got["rank"] == rank and got["world"] == 2
        assert got["total"] == 300.0  # units summed over ranks
        assert got["tmax"] == 1.5     # the slowest rank's time
        assert got["value"] == 200.0
        assert got["max_rank"] == 1.0


def test_single_process_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.dist_env() == (0, 1, 0) or "RANK" in os.environ
    assert bench.aggregate(42.0, 2.0) == (42.0, 2.0, 21.0)


@pytest.mark.timeout(300)
def test_reference_arm_as_two_ranks():
    port = _free_port()
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3"]
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=280)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout  # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0

"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The layer shards by independent token batches (one per GPU, weights
replicated), so the only cross-rank steps are the barrier and the
max-over-ranks reduction of the timed region; the reference arm runs on
rank 0 alone."""
import json
import os
import socket
import subprocess
import sys
from pathlib import Path

import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, str(ROOT))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
    got = bench.reduce_max(ms, dist, "cpu")
    dist.barrier()
    q.put((rank, got, bench.job_value(world, 64, 20, got)))
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]
    assert res[0][2] == pytest.approx(2 * 64 * 20 / 15e-3)


def test_single_rank_reduce_is_identity():
    sys.path.insert(0, str(ROOT))
    import bench
    assert bench.reduce_max(3.5) == 3.5
    assert bench.job_value(1, 64, 10, 1000.0) == pytest.approx(640.0)


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, str(ROOT / "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--steps", "2", "--warmup", "3"]
    out = subprocess.run(cmd, env=dict(env, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1"), capture_output=True,
                         text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""
    out = subprocess.run(cmd, env=dict(env, RANK="0", WORLD_SIZE="1"), capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def _ep_worker(rank, world, port, q):
    """The --ep mode's cross-rank steps on gloo: every rank times its own pass, the line takes
    the slowest rank's time and counts every rank's tokens."""
    import torch.distributed as dist
    sys.path.insert(0, str(ROOT))
    import bench
    from synth import workloads as W
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms = bench.reduce_max(4.0 + rank, dist, "cpu")
    e2e = bench.reduce_max(6.0 - rank, dist, "cpu")
    dist.barrier()
    line = bench.ep_line(world, W.WORKLOADS[1], 10, 3, ms, e2e, {}, 7)
    q.put((rank, json.dumps(line)))
    dist.destroy_process_group()


def test_expert_parallel_line_takes_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    lines = [json.loads(r[1]) for r in res]
    assert lines[0] == lines[1]
    line = lines[0]
    assert line["ms_per_step"] == pytest.approx(0.5)                     # max(4, 5) / 10 steps
    assert line["value"] == pytest.approx(2 * 64 * 10 / 5e-3)           # both ranks' tokens
    assert line["e2e"]["value"] == pytest.approx(2 * 64 * 10 / 6e-3)
    assert line["config"]["parallelism"].startswith("ep2 (64 experts per rank")
    assert line["gpu_launches"] == 70 and line["scaling"] == "weak"

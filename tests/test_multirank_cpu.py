"""The multi-process plumbing of bench.py on CPU: two gloo ranks (world size 2)
agree on the max-over-ranks time, draw different token batches for the same
weights, the reference arm runs on rank 0 only, and ``bench.py --gpus 2``
without a launcher starts two ranks itself and prints one line."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    import moe_inputs
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        spec = moe_inputs.CONFIGS["tiny"]
        seed = bench.rank_batch(spec, rank)
        x = moe_inputs.make_x(spec["T"], spec["H"], seed)
        t = bench.max_over_ranks(10.0 + rank, world)
        dist.barrier()
        q.put((rank, t, seed, float(x.float().sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert res[0][1] == res[1][1] == 11.0          # max over ranks
    assert res[0][2] != res[1][2]                  # each rank its own batch
    assert res[0][3] != res[1][3]


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_rank_behaviour(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "2", "--warmup", "1", "--gpus", "2"], capture_output=True, text=True, env=env,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    if rank == 0:
        assert len(lines) == 1
        d = json.loads(lines[0])
        assert d["impl"] == "reference" and d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0
        assert d["cpu_baseline"]["kind"] == "oracle"
    else:
        assert lines == []


def test_gpus_flag_launches_that_many_ranks():
    """`bench.py --gpus 2` with no launcher in the environment starts two
    ranks under torch.distributed.run (127.0.0.1); rank 0 alone prints, and
    the line reports both ranks."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR",
                                                             "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "2", "--warmup", "1", "--gpus", "2"], capture_output=True, text=True, env=env,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["impl"] == "reference"
    assert d["cpu_baseline"]["cores"] >= 1


def test_gpus_flag_must_match_the_launcher():
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "1", "--warmup", "1", "--gpus", "4"], capture_output=True, text=True, env=env,
                       timeout=120)
    assert r.returncode != 0
    assert "does not match WORLD_SIZE" in r.stderr

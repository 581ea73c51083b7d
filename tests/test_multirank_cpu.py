"""Multi-rank plumbing of bench.py on the CPU: two gloo ranks.

The layer has no cross-GPU exchange (tokens are independent, weights are
replicated), so ranks run replicas; the only collectives are the barrier and
the max-over-ranks of the device timings.  These tests run those helpers in
two real processes over gloo.
"""

import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = bench.dist_env()
        seconds = 0.5 + rank  # rank 1 is the slow one
        bench.barrier()
        slowest = bench.reduce_max(seconds)
        units = 1000.0
        agg = bench.aggregate(units, w, slowest)
        seed = bench.rank_seed(1, rank)
        bench.barrier()
        q.put((rank, r, w, lr, slowest, agg, seed))
    finally:
        dist.destroy_process_group()


def _run(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out)


def test_two_gloo_ranks_take_the_max_and_aggregate():
    out = _run(2)
    for rank, r, w, lr, slowest, agg, seed in out:
        assert (r, w, lr) == (rank, 2, rank)
        assert slowest == pytest.approx(1.5)  # every rank sees the slowest rank's time
        assert agg == pytest.approx(2 * 1000.0 / 1.5)  # all ranks' units over that time
    seeds = [o[-1] for o in out]
    assert seeds[0] == 1 and len(set(seeds)) == 2  # rank 0 keeps the workload's seed, ranks differ


def test_single_process_helpers_are_identities():
    assert bench.reduce_max(3.25) == 3.25
    assert bench.aggregate(10.0, 1, 2.0) == 5.0
    assert bench.rank_seed(7, 0) == 7
    bench.barrier()  # no process group: a no-op


def _bench(argv, timeout=300):
    import subprocess

    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + argv, capture_output=True, text=True,
                          timeout=timeout, env=env, cwd=ROOT)


def test_plain_launch_with_several_gpus_starts_one_rank_each():
    """`bench.py --gpus 2` run as a plain process starts two ranks under torch.distributed.run;
    the reference arm needs no GPU, so the whole launch runs here: rank 0 prints the one line,
    with n_gpus = 2."""
    import json

    r = _bench(["--gpus", "2", "--impl", "reference", "--workload", "cfg1", "--steps", "1", "--warmup", "3",
                "--cpu-budget", "0.5"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["n_gpus"] == 2


def test_plain_launch_refuses_more_gpus_than_visible():
    """Our arm with more ranks than visible GPUs fails loudly instead of measuring one replica."""
    r = _bench(["--gpus", "2", "--steps", "1", "--warmup", "3"], timeout=120)
    assert r.returncode != 0
    assert "CUDA device" in r.stderr
    assert "{" not in r.stdout


def test_relaunch_command_names_every_rank_and_the_loopback_address():
    cmd = bench.relaunch_command(4, ["--gpus", "4", "--steps", "5"], 29500)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd and "--master-port=29500" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "5"]

"""The benchmark's multi-rank host logic, on CPU with world size 2 over gloo.

The forward shards by sequence: each rank runs an independent replica on its
own batch, and the only collective is the max of the ranks' device times.
These tests run that logic in two gloo processes, and run the reference arm
under torchrun with two ranks (rank 0 alone prints its line)."""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

torch = pytest.importorskip("torch")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 2.0 + 3.0 * rank                                   # rank 1 is the slow one
        slow = bench.max_over_ranks(ms, world, "cpu")
        wl = bench.replica_workload(synth.WORKLOADS["c1"], rank, world)
        seeds = [None] * world
        dist.all_gather_object(seeds, wl.seed)
        out.put((rank, slow, bench.job_tokens_per_s(wl.n_tok, world, slow), seeds))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    n_tok = 256                                                  # c1: B=1, T=256 per replica
    for rank, slow, value, seeds in res:
        assert slow == 5.0                                       # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * n_tok / 5e-3)          # all ranks' tokens over that time
        assert len(set(seeds)) == 2                              # each replica draws its own batch


def test_single_rank_helpers_need_no_process_group():
    import bench
    import synth
    assert bench.max_over_ranks(3.5, 1) == 3.5
    wl = synth.WORKLOADS["c2"]
    assert bench.replica_workload(wl, 0, 1) is wl
    assert bench.job_tokens_per_s(16384, 1, 1.0) == pytest.approx(16384e3)


def test_reference_arm_two_ranks_prints_one_line():
    """torchrun with two CPU ranks: rank 0 times the oracle on a small sample
    and prints the contract's line; rank 1 exits 0 without work."""
    import oracle
    oracle.build()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "c1", "--ref-tokens", "8"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0

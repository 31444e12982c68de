"""The host logic of the sharded tables, on CPU: gloo ranks exchange their
shard exports and each maps the others' (fake export/open functions stand in
for CUDA IPC, which needs a GPU; the kernels' side is in
test_gpu_sharded.py)."""

import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

torch = pytest.importorskip("torch")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _fake_export(rank):
    def export(ptr):
        return bytes([rank]) * 64, ptr % 4096
    return export


def _fake_open(handle, offset):
    # a mapping of rank r's allocation lands at 10^6 * (r + 1); the pointer is base + offset
    base = 1_000_000 * (handle[0] + 1)
    return base + offset, base


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import hashed_gram_embedding_02_b200 as eb
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        def all_gather(obj):
            every = [None] * world
            dist.all_gather_object(every, obj)
            return every
        local = 4096 * 7 + 16 * (rank + 1)             # this rank's shard pointer
        ptrs, bases = eb.exchange_shards(local, rank, world, all_gather, _fake_export(rank), _fake_open)
        out.put((rank, ptrs, bases))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_shards_gloo(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ptrs, bases in res:
        assert len(ptrs) == world
        for g in range(world):
            off = 16 * (g + 1)
            want = 4096 * 7 + off if g == rank else 1_000_000 * (g + 1) + off
            assert ptrs[g] == want, (rank, g)
        assert sorted(bases) == sorted(1_000_000 * (g + 1) for g in range(world) if g != rank)


def test_exchange_shards_single_rank_maps_nothing():
    import hashed_gram_embedding_02_b200 as eb

    def fail(*a):
        raise AssertionError("no export or mapping with one rank")
    ptrs, bases = eb.exchange_shards(1234, 0, 1, fail, fail, fail)
    assert ptrs == [1234] and bases == []


def test_exchange_shards_rejects_a_short_gather():
    import hashed_gram_embedding_02_b200 as eb
    with pytest.raises(RuntimeError):
        eb.exchange_shards(16, 0, 3, lambda obj: [obj, obj], _fake_export(0), _fake_open)

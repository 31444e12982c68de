"""The backward's exchange of (row, gradient) pairs between ranks, on CPU:
gloo ranks run the package's all_to_all_pairs on segments routed here with
numpy (a stand-in for engram_grad_route, which needs a GPU; its side is in
test_gpu_grad_exchange.py).  Each rank must receive, from every rank in rank
order, exactly the segment that rank addressed to it, and the per-row sums
of what it received must equal the sums over all ranks' pairs of its rows
(integer-valued gradients, so every sum is exact).  Then the package's
sharded_table_step on two gloo ranks, with numpy stand-ins for the library
calls: each rank's shard must end as the whole table updated by the union
batch's gradient."""

import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

torch = pytest.importorskip("torch")

R_TOTAL, D = 997, 4


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _per(world):
    return (R_TOTAL + world - 1) // world


def _pairs(rank, world):
    """Rank `rank`'s distinct rows and integer-valued fp32 gradients (the last
    rank of three sends nothing at all)."""
    if world == 3 and rank == 2:
        return np.zeros(0, np.int64), np.zeros((0, D), np.float32)
    rng = np.random.default_rng(100 * world + rank)
    rows = rng.choice(R_TOTAL, size=40 + 15 * rank, replace=False).astype(np.int64)
    grad = rng.integers(-8, 9, size=(len(rows), D)).astype(np.float32)
    return rows, grad


def _route(rank, world):
    """Segments in owner order, shuffled inside each segment (as the device's atomics may)."""
    rows, grad = _pairs(rank, world)
    owner = rows // _per(world)
    rng = np.random.default_rng(7 + rank)
    order = np.concatenate([rng.permutation(np.flatnonzero(owner == g)) for g in range(world)]).astype(np.int64)
    counts = np.bincount(owner, minlength=world).astype(np.int64)
    # spare capacity past the pairs, as the device's send buffers have
    cap = len(rows) + 3
    send_rows = np.full(cap, -1, np.int64)
    send_grad = np.full((cap, D), np.nan, np.float32)
    send_rows[:len(rows)] = rows[order]
    send_grad[:len(rows)] = grad[order]
    return send_rows, send_grad, counts


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import hashed_gram_embedding_02_b200 as eb
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sr, sg, sc = _route(rank, world)
        rr, rg, counts = eb.all_to_all_pairs(torch.from_numpy(sr), torch.from_numpy(sg), torch.from_numpy(sc))
        out.put((rank, rr.numpy(), rg.numpy(), counts))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_all_to_all_pairs_gloo(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    res = sorted((q.get(timeout=120) for _ in ps), key=lambda x: x[0])
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    routed = [_route(r, world) for r in range(world)]
    for g, rr, rg, counts in res:
        # from every rank, in rank order, the segment it addressed to g
        want_r, want_g, want_c = [], [], []
        for sr, sg, sc in routed:
            off = int(sc[:g].sum())
            want_r.append(sr[off:off + sc[g]])
            want_g.append(sg[off:off + sc[g]])
            want_c.append(int(sc[g]))
        assert counts == want_c
        assert np.array_equal(rr, np.concatenate(want_r))
        assert np.array_equal(rg, np.concatenate(want_g))
        # every row of g's range, summed over the ranks' pairs
        lo, hi = g * _per(world), min(R_TOTAL, (g + 1) * _per(world))
        assert ((rr >= lo) & (rr < hi)).all()
        total = np.zeros((R_TOTAL, D), np.float64)
        for r in range(world):
            rows, grad = _pairs(r, world)
            np.add.at(total, rows, grad)
        got = np.zeros((R_TOTAL, D), np.float64)
        np.add.at(got, rr, rg)
        assert np.array_equal(got[lo:hi], total[lo:hi])


def test_all_to_all_pairs_single_rank_is_a_copy():
    import hashed_gram_embedding_02_b200 as eb
    calls = []

    def a2a(out, inp, out_split=None, in_split=None):
        calls.append((out_split, in_split))
        out.copy_(inp)

    sr, sg, sc = _route(0, 1)
    rr, rg, counts = eb.all_to_all_pairs(torch.from_numpy(sr), torch.from_numpy(sg), torch.from_numpy(sc), a2a)
    n = int(sc[0])
    assert counts == [n] and calls == [(None, None), ([n], [n]), ([n], [n])]
    assert np.array_equal(rr.numpy(), sr[:n]) and np.array_equal(rg.numpy(), sg[:n])


def test_all_to_all_pairs_rejects_bad_counts():
    import hashed_gram_embedding_02_b200 as eb

    def a2a(out, inp, out_split=None, in_split=None):
        out.copy_(inp)

    rows = torch.zeros(4, dtype=torch.int64)
    grad = torch.zeros(4, D)
    with pytest.raises(RuntimeError):   # more pairs than the send buffers hold
        eb.all_to_all_pairs(rows, grad, torch.tensor([5], dtype=torch.int64), a2a)
    with pytest.raises(RuntimeError):   # a negative count
        eb.all_to_all_pairs(rows, grad, torch.tensor([-1], dtype=torch.int64), a2a)


# ------------------------------------------------- the whole step, two ranks

J_T, M_T, D_T, N_T = 2, 11, 3, 9          # 2 tables of 11 rows of width 3; 9 tokens per rank


def _batch(rank):
    rng = np.random.default_rng(40 + rank)
    idx = rng.integers(0, M_T, size=(N_T, J_T)).astype(np.uint32)
    de = rng.integers(-4, 5, size=(N_T, J_T * D_T)).astype(np.float64)
    return idx, de


class _HostEngram:
    """Stand-ins for the library calls sharded_table_step makes, in numpy,
    with the oracle's gradient: the step's wiring and its exchange are what
    is tested here (the kernels are tested on the GPU)."""

    def __init__(self, world):
        self.world = world
        self.R = J_T * M_T
        self.per = (self.R + world - 1) // world

    def table_grad(self, idx, d_e):
        import oracle
        keys, grad = oracle.table_grad(idx.numpy(), np.full(J_T, M_T, np.uint32), d_e.numpy(), D_T)
        return torch.from_numpy(keys.astype(np.int64)), torch.from_numpy(grad), torch.tensor([len(keys)])

    def grad_route(self, rows, grad, n_pairs, n_shards):
        owner = rows.numpy() // self.per
        order = np.argsort(owner, kind="stable")
        counts = np.bincount(owner, minlength=n_shards).astype(np.int64)
        return rows[order].contiguous(), grad[order].contiguous(), torch.from_numpy(counts)

    def grad_combine(self, pair_rows, pair_grad, n_shards, shard):
        got = {}
        for r, g in zip(pair_rows.tolist(), pair_grad.numpy()):
            assert r // self.per == shard
            got[r] = got.get(r, 0) + g
        keys = sorted(got)
        grad = np.array([got[k] for k in keys]).reshape(len(keys), D_T)
        return torch.tensor(keys, dtype=torch.int64), torch.from_numpy(grad), torch.tensor([len(keys)])

    def shard_sgd(self, n_shards, shard, rows, grad, n_unique, shard_table, lr):
        first = shard * self.per
        for r, g in zip(rows.tolist(), grad):
            shard_table[r - first] -= lr * g


def _full_table():
    return np.arange(J_T * M_T * D_T, dtype=np.float64).reshape(J_T * M_T, D_T) / 7.0


def _step_main(rank, world, port, out):
    import datetime
    import types

    import torch.distributed as dist

    import hashed_gram_embedding_02_b200 as eb
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        eng = _HostEngram(world)
        lo, hi = rank * eng.per, min(eng.R, (rank + 1) * eng.per)
        shards = types.SimpleNamespace(local=torch.from_numpy(_full_table()[lo:hi].copy()))
        idx, de = _batch(rank)
        eb.sharded_table_step(eng, shards, torch.from_numpy(idx), torch.from_numpy(de), 0.5, rank, world)
        out.put((rank, lo, shards.local.numpy()))
    finally:
        dist.destroy_process_group()


def test_sharded_table_step_two_ranks_gloo():
    import torch.multiprocessing as mp

    import oracle
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_step_main, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    res = sorted((q.get(timeout=120) for _ in ps), key=lambda x: x[0])
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the full table after one step on the union of the two batches
    idx = np.concatenate([_batch(r)[0] for r in range(world)])
    de = np.concatenate([_batch(r)[1] for r in range(world)])
    keys, grad = oracle.table_grad(idx, np.full(J_T, M_T, np.uint32), de, D_T)
    want = _full_table()
    want[keys.astype(np.int64)] -= 0.5 * grad
    for rank, lo, shard in res:
        np.testing.assert_array_equal(shard, want[lo:lo + len(shard)])
    assert sum(len(s) for _, _, s in res) == J_T * M_T

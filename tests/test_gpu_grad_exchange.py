"""The tables' backward across shards, on one GPU with the ranks emulated in
one process.

Every emulated rank takes the sparse gradient of its own batch
(engram_table_grad) and routes it to the shards that own the rows
(engram_grad_route).  The exchange is emulated by what an all-to-all leaves
on each owner: the segments the ranks sent it, concatenated in rank order.
Each shard then sums its pairs per row (engram_grad_combine) and updates its
rows (engram_shard_sgd).

Checked against the oracle's gradient of the union of the ranks' batches on
each shard's rows: the distinct rows exactly, each sum within the bound of
fp32 summation of its k lookups in any order, (k - 1) * 2^-24 * sum |x|
(Higham, Accuracy and Stability of Numerical Algorithms, 2nd ed., section
4.2), plus one rounding.  The combine must not depend on the order inside a
rank's segment (bit for bit), and the shard update must equal the full-table
update with the same pairs (bit for bit)."""

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import config_for

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
CASES = {
    "bf16": W["c1"].replace(name="x1", B=2, T=160, K=4, D=64, d=256, dtype="bf16", seed=81),
    "fp32": W["c1"].replace(name="x2", B=2, T=100, seed=82),
}


@pytest.fixture(scope="module")
def eb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hashed_gram_embedding_02_b200 as eb
    return eb


def _rank_batch(eb, ctx, inp, rank):
    """Rank `rank`'s idx and dL/de: its own Zipf tokens, the shared remap and hash."""
    wl = inp.wl
    tok = synth.zipf_tokens(wl.replace(seed=wl.seed + 1000 * rank))
    idx = torch.empty(wl.n_tok, wl.J, dtype=torch.int32, device="cuda")
    eb.engram_hash(ctx.ctx, torch.from_numpy(tok).cuda(), torch.from_numpy(inp.P).cuda(), wl.B, wl.T, wl.T,
                   wl.t_begin, idx)
    g = torch.Generator(device="cuda").manual_seed(500 + rank)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    de = (torch.randn(wl.n_tok, wl.d_mem, device="cuda", generator=g) * 0.01).to(dt)
    return idx, de


def _by_row(rows, grad):
    r = rows.cpu().numpy().astype(np.int64)
    o = np.argsort(r)
    return r[o], grad.cpu().numpy()[o]


def _segments(send_rows, send_grad, counts):
    """[(rows, grad)] of every destination shard, in shard order."""
    out, off = [], 0
    for c in counts:
        out.append((send_rows[off:off + c], send_grad[off:off + c]))
        off += c
    return out


def _route_all(eb, ctx, inp, G):
    """Every rank's pairs, its routed segments and its batch."""
    ranks = []
    for r in range(G):
        idx, de = _rank_batch(eb, ctx, inp, r)
        rows, grad, cnt = ctx.table_grad(idx, de)
        send_rows, send_grad, send_counts = ctx.grad_route(rows, grad, cnt, G)
        torch.cuda.synchronize()
        counts = [int(x) for x in send_counts.cpu().tolist()]
        ranks.append(dict(idx=idx, de=de, rows=rows, grad=grad, counts=counts,
                          seg=_segments(send_rows, send_grad, counts)))
    return ranks


def _received(ranks, g, reverse=False):
    """What the all-to-all leaves on shard g: the ranks' segments for g in rank order."""
    rows = [rk["seg"][g][0] for rk in ranks]
    grad = [rk["seg"][g][1] for rk in ranks]
    if reverse:   # another order inside every rank's segment
        rows = [x.flip(0) for x in rows]
        grad = [x.flip(0) for x in grad]
    return torch.cat(rows).contiguous(), torch.cat(grad).contiguous()


@pytest.mark.parametrize("name,G", [("bf16", 2), ("bf16", 3), ("bf16", 5), ("fp32", 2)])
def test_sharded_backward_matches_the_union_gradient(eb, name, G):
    wl = CASES[name]
    inp = synth.Inputs(wl)
    ctx = eb.Engram(config_for(inp, eb))
    ranks = _route_all(eb, ctx, inp, G)
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    bounds = [eb.engram_shard_range(ctx.ctx, G, g) for g in range(G)]

    # routing: every rank sends each of its pairs once, to the shard that owns the row, unchanged
    for rk in ranks:
        r_all, g_all = _by_row(rk["rows"], rk["grad"])
        got_r, got_g = [], []
        for g, (lo, n) in enumerate(bounds):
            sr, sg = rk["seg"][g]
            sr_np = sr.cpu().numpy()
            assert rk["counts"][g] == int(((r_all >= lo) & (r_all < lo + n)).sum())
            assert ((sr_np >= lo) & (sr_np < lo + n)).all()
            got_r.append(sr)
            got_g.append(sg)
        r2, g2 = _by_row(torch.cat(got_r), torch.cat(got_g))
        assert np.array_equal(r2, r_all) and np.array_equal(g2, g_all)

    # the union of the batches, as the oracle sees it
    idx_np = np.concatenate([rk["idx"].cpu().numpy().view(np.uint32) for rk in ranks])
    de_np = np.concatenate([rk["de"].float().cpu().numpy().astype(np.float64) for rk in ranks])
    keys, ref = oracle.table_grad(idx_np, inp.rows, de_np, wl.D)
    _, absum = oracle.table_grad(idx_np, inp.rows, np.abs(de_np), wl.D)
    _, cnt = oracle.table_grad(idx_np, inp.rows, np.ones_like(de_np), wl.D)
    keys = np.asarray(keys, dtype=np.int64)

    tables = inp.device_tables("cuda:0").reshape(-1, wl.D)
    lr = 0.25
    total = 0
    for g, (lo, n) in enumerate(bounds):
        pr, pg = _received(ranks, g)
        rows, grad, u = ctx.grad_combine(pr, pg, G, g)
        torch.cuda.synchronize()
        assert ctx.status() == (eb.ENGRAM_OK, 0)
        r, s = _by_row(rows, grad)
        sel = (keys >= lo) & (keys < lo + n)
        assert np.array_equal(r, keys[sel]), g
        bound = np.maximum(cnt[sel] - 1, 0) * 2.0 ** -24 * absum[sel] + 2.0 ** -24 * np.abs(ref[sel]) + 1e-38
        err = np.abs(s - ref[sel])
        assert not (err > bound).any(), (g, int((err > bound).sum()), float(err.max()))
        total += len(r)

        # the order inside a rank's segment changes nothing
        rows2, grad2, _ = ctx.grad_combine(*_received(ranks, g, reverse=True), G, g)
        r2, s2 = _by_row(rows2, grad2)
        assert np.array_equal(r2, r) and np.array_equal(s2, s)

        # the shard's update equals the full-table update with the same pairs
        shard = tables[lo:lo + n].clone()
        full = tables.clone()
        ctx.shard_sgd(G, g, rows, grad, u, shard, lr)
        eb.engram_table_sgd(ctx.ctx, rows, grad, u, rows.shape[0], full, lr)
        torch.cuda.synchronize()
        assert ctx.status() == (eb.ENGRAM_OK, 0)
        assert torch.equal(shard, full[lo:lo + n]), g
        assert torch.equal(full[:lo], tables[:lo]) and torch.equal(full[lo + n:], tables[lo + n:])
    assert total == len(keys)


def test_combine_drops_pairs_of_other_shards_and_empty_input(eb):
    wl = CASES["bf16"]
    inp = synth.Inputs(wl)
    ctx = eb.Engram(config_for(inp, eb))
    G = 2
    ranks = _route_all(eb, ctx, inp, G)
    pr0, pg0 = _received(ranks, 0)
    pr1, pg1 = _received(ranks, 1)
    assert len(pr0) and len(pr1)
    ctx.status()
    # shard 0 given its own pairs plus one of shard 1's: that one is flagged and dropped
    rows, grad, _ = ctx.grad_combine(torch.cat([pr0, pr1[:1]]), torch.cat([pg0, pg1[:1]]).contiguous(), G, 0)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_E_DEVICE, eb.ENGRAM_ERR_INDEX)
    want_r, want_g = _by_row(*ctx.grad_combine(pr0, pg0, G, 0)[:2])
    r, s = _by_row(rows, grad)
    assert np.array_equal(r, want_r) and np.array_equal(s, want_g)
    # nothing received: no rows, and an update of nothing
    empty_r = torch.empty(0, dtype=torch.int64, device="cuda")
    empty_g = torch.empty(0, wl.D, dtype=torch.float32, device="cuda")
    rows, grad, u = ctx.grad_combine(empty_r, empty_g, G, 1)
    assert rows.numel() == 0 and int(u.item()) == 0
    lo, n = eb.engram_shard_range(ctx.ctx, G, 1)
    shard = inp.device_tables("cuda:0").reshape(-1, wl.D)[lo:lo + n].clone()
    before = shard.clone()
    ctx.shard_sgd(G, 1, rows, grad, u, shard, 0.5)
    torch.cuda.synchronize()
    assert torch.equal(shard, before)
    assert ctx.status() == (eb.ENGRAM_OK, 0)


def test_route_flags_rows_beyond_the_tables(eb):
    wl = CASES["bf16"]
    inp = synth.Inputs(wl)
    ctx = eb.Engram(config_for(inp, eb))
    R = int(np.sum(inp.rows.astype(np.int64)))
    rows = torch.tensor([3, R + 5, R - 1], dtype=torch.int64, device="cuda")
    grad = torch.arange(3 * wl.D, dtype=torch.float32, device="cuda").reshape(3, wl.D)
    cnt = torch.tensor([3], dtype=torch.int64, device="cuda")
    send_rows, send_grad, send_counts = ctx.grad_route(rows, grad, cnt, 2)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_E_DEVICE, eb.ENGRAM_ERR_INDEX)
    assert send_counts.cpu().tolist() == [1, 1]
    assert send_rows[:2].cpu().tolist() == [3, R - 1]
    assert torch.equal(send_grad[0], grad[0]) and torch.equal(send_grad[1], grad[2])


def test_sharded_table_step_on_one_rank(eb):
    """The whole step through the package's plumbing, with one rank (the
    exchange is then a copy): it must equal engram_table_grad followed by
    engram_table_sgd on the whole table."""
    wl = CASES["bf16"]
    inp = synth.Inputs(wl)
    ctx = eb.Engram(config_for(inp, eb))
    full = inp.device_tables("cuda:0").reshape(-1, wl.D)

    def fill(first, n, out):
        out.copy_(full[first:first + n])

    shards = eb.ShardedTables(ctx, 1, 0, wl.D, full.dtype, torch.device("cuda:0"), fill)

    def a2a(out, inp_, out_split=None, in_split=None):
        out.copy_(inp_)

    idx, de = _rank_batch(eb, ctx, inp, 0)
    rows, grad = eb.sharded_table_step(ctx, shards, idx, de, 0.5, 0, 1, all_to_all_single=a2a)
    r0, g0, c0 = ctx.table_grad(idx, de)
    want = full.clone()
    eb.engram_table_sgd(ctx.ctx, r0, g0, c0, r0.shape[0], want, 0.5)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    a, b = _by_row(rows, grad)
    a0, b0 = _by_row(r0, g0)
    assert np.array_equal(a, a0) and np.array_equal(b, b0)
    assert torch.equal(shards.local, want)
    shards.close()

"""Host-memory tier on the GPU: the rows fetched from host tables over PCIe
and gathered from the staging buffer must equal, bit for bit, the gather
from the same tables in HBM; the distinct-row count must equal the number of
distinct (table, row) lookups; and the forward on top matches the oracle."""

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import DeviceInputs, bf16_bound, config_for, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
# 256-byte rows as at the host-memory configuration, small tables
SMALL = W["c5"].replace(name="h1", B=2, T=700, M=100003, d=512, seed=21)
# the host-memory configuration's batch (8 x 4096 tokens, 524288 lookups) on 1000003-row tables
FULL_BATCH = W["c5"].replace(name="h2", M=1000003, seed=22)


@pytest.fixture(scope="module")
def eb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hashed_gram_embedding_02_b200 as eb
    return eb


def _indices(eb, ctx, di, wl):
    idx = torch.empty(wl.n_tok, wl.J, dtype=torch.int32, device="cuda")
    eb.engram_hash(ctx.ctx, di.tok, di.P, wl.B, wl.T, wl.T, 0, idx)
    return idx


def _distinct_rows(idx, inp):
    off = np.concatenate([[0], np.cumsum(inp.rows[:-1].astype(np.int64))])
    ix = idx.cpu().numpy().view(np.uint32).astype(np.int64)
    valid = ix < inp.rows[None, :].astype(np.int64)
    return len(np.unique((ix + off[None, :])[valid]))


def _staged_e(eb, ctx, tier, idx, wl, side):
    e = torch.full((wl.n_tok, wl.d_mem), float("nan"), dtype=torch.bfloat16, device="cuda")
    tier.dedupe(idx, wl.n_tok)
    n_unique = tier.fetch(side)
    tier.gather(wl.n_tok, e)
    torch.cuda.synchronize()
    return e, n_unique


@pytest.mark.parametrize("wl", [SMALL, FULL_BATCH], ids=["small", "c5_batch"])
def test_staged_gather_equals_hbm_gather(eb, wl):
    inp = synth.Inputs(wl)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    host = inp.host_tables("cuda:0")
    tier = eb.HostTier(ctx, host, max_lookups=wl.n_tok * wl.J, n_threads=8)
    idx = _indices(eb, ctx, di, wl)
    side = torch.cuda.Stream()
    e_t, n_unique = _staged_e(eb, ctx, tier, idx, wl, side)
    e_d = torch.empty_like(e_t)
    eb.engram_gather(ctx.ctx, idx, wl.n_tok, di.tables, e_d)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    assert torch.equal(e_t, e_d)
    assert n_unique == _distinct_rows(idx, inp)
    assert n_unique < wl.n_tok * wl.J                      # Zipf n-grams repeat
    st = tier.stats()
    assert st["n_unique"] == n_unique and st["n_copies"] >= 1 and st["copy_ms"] > 0


def test_consecutive_batches_reuse_the_buffers(eb):
    wl = SMALL
    ctx_inputs = [synth.Inputs(wl.replace(seed=wl.seed + k)) for k in range(3)]
    ctx = eb.Engram(config_for(ctx_inputs[0], eb))
    host = ctx_inputs[0].host_tables("cuda:0")          # tables depend on the seed: use batch 0's for all
    tables_d = ctx_inputs[0].device_tables("cuda:0")
    tier = eb.HostTier(ctx, host, max_lookups=wl.n_tok * wl.J, n_threads=4)
    side = torch.cuda.Stream()
    for inp in ctx_inputs:
        di_tok = torch.from_numpy(inp.tok).cuda()
        P = torch.from_numpy(inp.P).cuda()
        idx = torch.empty(wl.n_tok, wl.J, dtype=torch.int32, device="cuda")
        eb.engram_hash(ctx.ctx, di_tok, P, wl.B, wl.T, wl.T, 0, idx)
        e_t = torch.empty(wl.n_tok, wl.d_mem, dtype=torch.bfloat16, device="cuda")
        tier.dedupe(idx, wl.n_tok)
        tier.fetch(side)
        tier.gather(wl.n_tok, e_t)
        e_d = torch.empty_like(e_t)
        eb.engram_gather(ctx.ctx, idx, wl.n_tok, tables_d, e_d)
        torch.cuda.synchronize()
        assert torch.equal(e_t, e_d)


def test_invalid_tokens_are_not_fetched(eb):
    wl = SMALL
    inp = synth.Inputs(wl)
    inp.tok[0, :] = wl.V + 1                             # a whole sequence of invalid ids
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    tier = eb.HostTier(ctx, inp.host_tables("cuda:0"), max_lookups=wl.n_tok * wl.J, n_threads=2)
    idx = _indices(eb, ctx, di, wl)
    side = torch.cuda.Stream()
    e_t, n_unique = _staged_e(eb, ctx, tier, idx, wl, side)
    st, flags = ctx.status()
    assert flags & eb.ENGRAM_ERR_TOKEN and not flags & eb.ENGRAM_ERR_INDEX
    assert n_unique == _distinct_rows(idx, inp)
    assert float(e_t[: wl.T].float().abs().max()) == 0.0   # sequence 0: every n-gram has an invalid id
    e_d = torch.empty_like(e_t)
    eb.engram_gather(ctx.ctx, idx, wl.n_tok, di.tables, e_d)
    torch.cuda.synchronize()
    assert torch.equal(e_t, e_d)


def test_forward_through_the_host_tier_matches_oracle(eb):
    wl = SMALL
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    tier = eb.HostTier(ctx, inp.host_tables("cuda:0"), max_lookups=wl.n_tok * wl.J, n_threads=8)
    idx = _indices(eb, ctx, di, wl)
    side = torch.cuda.Stream()
    e_t, _ = _staged_e(eb, ctx, tier, idx, wl, side)
    ws_bytes = eb.engram_workspace_bytes(ctx.ctx, wl.B, wl.T)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    y = di.empty_y()
    eb.engram_gate_conv(ctx.ctx, e_t, di.h, di.Wk, di.Wv, di.gq, di.gk, di.conv_w, wl.B, wl.T, None, y, None, 1,
                        ws, ws_bytes)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    pos = synth.sample_positions(wl, 64, seed=3)
    ref = oracle.forward_rows(inp, pos, add_residual=True)
    y_s = to_np(y[torch.from_numpy(pos).cuda()])
    err = np.abs(y_s - ref.y)
    assert err.max() <= 2e-2
    assert not (err > bf16_bound(ref.y, ref.vt_win, inp.conv_w)).any()


def test_host_tier_rejects_batches_beyond_its_capacity(eb):
    wl = SMALL
    inp = synth.Inputs(wl)
    ctx = eb.Engram(config_for(inp, eb))
    host = torch.zeros(wl.J, inp.M, wl.D, dtype=torch.bfloat16)
    tier = eb.HostTier(ctx, host, max_lookups=100 * wl.J, n_threads=1)
    idx = torch.zeros(101, wl.J, dtype=torch.int32, device="cuda")
    with pytest.raises(eb.EngramError):
        tier.dedupe(idx, 101)
    with pytest.raises(eb.EngramError):
        tier.fetch(torch.cuda.Stream())                  # no dedupe yet


def test_c5_batch_forward_sampled_matches_oracle(eb):
    """The host-memory configuration's batch (8 x 4096 tokens, d_mem 2048)
    through dedupe, fetch, staged gather and the fused passes, checked
    against the oracle at sampled rows (first rows, sequence ends included)."""
    wl = FULL_BATCH
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    tier = eb.HostTier(ctx, inp.host_tables("cuda:0"), max_lookups=wl.n_tok * wl.J, n_threads=8)
    idx = _indices(eb, ctx, di, wl)
    e_t, _ = _staged_e(eb, ctx, tier, idx, wl, torch.cuda.Stream())
    ws_bytes = eb.engram_workspace_bytes(ctx.ctx, wl.B, wl.T)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    y = di.empty_y()
    alpha = torch.empty(wl.n_tok, dtype=torch.float32, device="cuda")
    eb.engram_gate_conv(ctx.ctx, e_t, di.h, di.Wk, di.Wv, di.gq, di.gk, di.conv_w, wl.B, wl.T, None, y, alpha, 1,
                        ws, ws_bytes)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    canon_ref, _ = oracle.remap(inp.tok, inp.P)
    idx_ref, _ = oracle.hash_ids(canon_ref, wl.Vc, wl.orders, wl.K, inp.mult, inp.rows)
    assert np.array_equal(idx.cpu().numpy().view(np.uint32), idx_ref)
    pos = synth.sample_positions(wl, 96, seed=9)
    ref = oracle.forward_rows(inp, pos, add_residual=True, idx=idx_ref)
    sel = torch.from_numpy(pos).cuda()
    np.testing.assert_allclose(to_np(alpha[sel]), ref.alpha, rtol=0, atol=2e-6)
    y_s = to_np(y[sel])
    err = np.abs(y_s - ref.y)
    assert err.max() <= 2e-2
    assert not (err > bf16_bound(ref.y, ref.vt_win, inp.conv_w)).any()


# ---------------------------------------------------------------- failure paths (made on the host)

@pytest.mark.parametrize("inject,status", [("list", "timeout"), ("pack", "host")])
def test_fetch_failure_is_reported_and_the_tier_recovers(eb, inject, status):
    """A host-side fault of one fetch: the distinct-row list that never
    arrives (the event query's answer is faked), or a packing thread that
    abandons the batch's last chunk.  The fetch returns ENGRAM_E_TIMEOUT or
    ENGRAM_E_HOST within a few seconds, gather_staged refuses the failed
    batch, and the next batch on the same tier matches the HBM gather bit for
    bit.  Nothing faults or stalls the GPU."""
    import time
    wl = SMALL
    inp = synth.Inputs(wl)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    host = inp.host_tables("cuda:0")
    # one thread: the abandoned chunk is the last one, after the earlier
    # chunks' copies were enqueued (their end must be recorded for the next fetch)
    tier = eb.HostTier(ctx, host, max_lookups=wl.n_tok * wl.J, n_threads=1)
    idx = _indices(eb, ctx, di, wl)
    side = torch.cuda.Stream()
    tier.debug(eb.ENGRAM_INJECT_LIST_WAIT if inject == "list" else eb.ENGRAM_INJECT_PACK_ABANDON, 1.0)
    tier.dedupe(idx, wl.n_tok)
    t0 = time.time()
    with pytest.raises(eb.EngramError) as err:
        tier.fetch(side)
    took = time.time() - t0
    want = eb.ENGRAM_E_TIMEOUT if status == "timeout" else eb.ENGRAM_E_HOST
    assert err.value.status == want
    assert 0.9 <= took < 10.0, took
    e = torch.empty(wl.n_tok, wl.d_mem, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(eb.EngramError) as err2:
        tier.gather(wl.n_tok, e)
    assert err2.value.status == eb.ENGRAM_E_INVAL
    # the next batch, same tier
    e_t, n_unique = _staged_e(eb, ctx, tier, idx, wl, side)
    e_d = torch.empty_like(e_t)
    eb.engram_gather(ctx.ctx, idx, wl.n_tok, di.tables, e_d)
    torch.cuda.synchronize()
    assert torch.equal(e_t, e_d)
    assert n_unique == _distinct_rows(idx, inp)
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    tier.close()


# ---------------------------------------------------------------- hot-row cache in HBM

def _batches(wl, n):
    """n token batches of the same workload (different seeds); the tables are batch 0's for all."""
    return [synth.Inputs(wl.replace(seed=wl.seed + k)) for k in range(n)]


def _distinct_split(idx, inp, cached_keys):
    off = np.concatenate([[0], np.cumsum(inp.rows[:-1].astype(np.int64))])
    ix = idx.cpu().numpy().view(np.uint32).astype(np.int64)
    valid = ix < inp.rows[None, :].astype(np.int64)
    keys, counts = np.unique((ix + off[None, :])[valid], return_counts=True)
    return keys, counts


@pytest.mark.parametrize("capacity", [60000, 500])
def test_hot_row_cache_over_batches(eb, capacity):
    """Five consecutive batches through a tier with a hot-row cache: each
    batch's staged gather equals the HBM gather bit for bit; fetched +
    cached rows = the batch's distinct rows; the first batch finds the cache
    empty and fetches everything; the cache fills with rows looked up at
    least twice, never beyond its capacity; later batches take rows from it;
    a reset empties it."""
    wl = SMALL
    batches = _batches(wl, 5)
    ctx = eb.Engram(config_for(batches[0], eb))
    host = batches[0].host_tables("cuda:0")
    tables_d = batches[0].device_tables("cuda:0")
    tier = eb.HostTier(ctx, host, max_lookups=wl.n_tok * wl.J, n_threads=4)
    tier.enable_cache(capacity, min_count=2)
    side = torch.cuda.Stream()
    admitted_possible = set()         # rows looked up >= 2 times in some earlier batch
    resident_prev = 0
    for k, inp in enumerate(batches):
        tok = torch.from_numpy(inp.tok).cuda()
        P = torch.from_numpy(inp.P).cuda()
        idx = torch.empty(wl.n_tok, wl.J, dtype=torch.int32, device="cuda")
        eb.engram_hash(ctx.ctx, tok, P, wl.B, wl.T, wl.T, 0, idx)
        e_t = torch.full((wl.n_tok, wl.d_mem), float("nan"), dtype=torch.bfloat16, device="cuda")
        tier.dedupe(idx, wl.n_tok)
        n_fetched = tier.fetch(side)
        tier.gather(wl.n_tok, e_t)
        e_d = torch.empty_like(e_t)
        eb.engram_gather(ctx.ctx, idx, wl.n_tok, tables_d, e_d)
        torch.cuda.synchronize()
        assert torch.equal(e_t, e_d), k
        keys, counts = _distinct_split(idx, batches[0], None)
        cs = tier.cache_stats()
        assert cs["capacity"] == capacity
        assert cs["fetched_rows"] == n_fetched
        assert cs["fetched_rows"] + cs["cached_rows"] == len(keys)
        assert cs["lookups"] == wl.n_tok * wl.J
        assert cs["resident"] >= resident_prev and cs["resident"] <= capacity
        if k == 0:
            assert cs["cached_rows"] == 0 and cs["resident"] == 0
        else:
            # every row served from the cache was a candidate of an earlier batch
            assert cs["cached_rows"] > 0
            assert cs["cached_rows"] <= len(set(keys.tolist()) & admitted_possible)
            assert cs["cached_lookups"] >= cs["cached_rows"]
        admitted_possible |= set(keys[counts >= 2].tolist())
        resident_prev = cs["resident"]
    if capacity == 500:
        assert resident_prev == 500
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    # a reset empties the cache: the next batch fetches every distinct row
    tier.reset_cache()
    inp = batches[1]
    idx = torch.empty(wl.n_tok, wl.J, dtype=torch.int32, device="cuda")
    eb.engram_hash(ctx.ctx, torch.from_numpy(inp.tok).cuda(), torch.from_numpy(inp.P).cuda(), wl.B, wl.T, wl.T, 0,
                   idx)
    e_t = torch.empty(wl.n_tok, wl.d_mem, dtype=torch.bfloat16, device="cuda")
    tier.dedupe(idx, wl.n_tok)
    tier.fetch(side)
    tier.gather(wl.n_tok, e_t)
    torch.cuda.synchronize()
    cs = tier.cache_stats()
    assert cs["cached_rows"] == 0 and cs["resident"] == 0
    e_d = torch.empty_like(e_t)
    eb.engram_gather(ctx.ctx, idx, wl.n_tok, tables_d, e_d)
    torch.cuda.synchronize()
    assert torch.equal(e_t, e_d)
    tier.close()


# ---------------------------------------------------------------- mapped fetch (GPU reads the host tables)

@pytest.mark.parametrize("cache", [0, 20000])
def test_mapped_fetch_equals_hbm_gather(eb, cache):
    """With the host tables mapped into the device's address space, a GPU
    kernel pulls the distinct rows over PCIe: three consecutive batches (with
    and without the hot-row cache) must gather exactly what the HBM gather
    gives, and the counts must match the copy path's."""
    wl = SMALL
    batches = _batches(wl, 3)
    ctx = eb.Engram(config_for(batches[0], eb))
    host = batches[0].host_tables("cuda:0")
    tables_d = batches[0].device_tables("cuda:0")
    tier = eb.HostTier(ctx, host, max_lookups=wl.n_tok * wl.J, n_threads=2)
    tier.map_tables()
    if cache:
        tier.enable_cache(cache)
    side = torch.cuda.Stream()
    for k, inp in enumerate(batches):
        idx = torch.empty(wl.n_tok, wl.J, dtype=torch.int32, device="cuda")
        eb.engram_hash(ctx.ctx, torch.from_numpy(inp.tok).cuda(), torch.from_numpy(inp.P).cuda(), wl.B, wl.T, wl.T,
                       0, idx)
        e_t = torch.full((wl.n_tok, wl.d_mem), float("nan"), dtype=torch.bfloat16, device="cuda")
        tier.dedupe(idx, wl.n_tok)
        assert tier.fetch(side) == -1                  # not known on the host at this point
        tier.gather(wl.n_tok, e_t)
        e_d = torch.empty_like(e_t)
        eb.engram_gather(ctx.ctx, idx, wl.n_tok, tables_d, e_d)
        torch.cuda.synchronize()
        assert torch.equal(e_t, e_d), k
        keys, _ = _distinct_split(idx, batches[0], None)
        cs = tier.cache_stats()
        assert cs["fetched_rows"] + cs["cached_rows"] == len(keys)
        st = tier.stats()
        assert st["n_unique"] == cs["fetched_rows"] and st["copy_ms"] > 0
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    tier.close()

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

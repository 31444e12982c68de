"""GPU path vs the oracle, element by element, through the C ABI.

Integer work (canonical ids, indices, gathered rows) must be bit-exact.  Gated
outputs: fp32 within max-abs 1e-5; bf16 within max-abs 2e-2 and within the
elementwise bound of gpu_helpers.bf16_bound.  Small workloads compare every
row; the full-size workloads compare every index and a seeded sample of
output rows (each sequence's first four and last rows included).
"""

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import DeviceInputs, bf16_bound, config_for, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
# small workloads that the oracle runs in full (ragged row counts on purpose)
SMALL = {
    "c1": W["c1"],
    # bf16, tensor-core tiling (d % 128 == 0, d_mem % 64 == 0), 400 rows
    "b1": W["c1"].replace(name="b1", B=2, T=200, K=4, D=64, d=256, dtype="bf16", seed=11),
    # bf16 on the CUDA-core projection (d not a multiple of 128), 64-byte rows, w = 3
    "b2": W["c1"].replace(name="b2", B=3, T=61, K=2, D=32, d=264, w=3, dtype="bf16", seed=12),
    # fp32, ragged everything, w = 2, single order
    "f2": W["c1"].replace(name="f2", B=3, T=77, orders=(3,), K=3, D=8, d=136, w=2, seed=13),
    # bf16 tensor-core tiling with several row tiles and a ragged tail, d_mem 1024
    "b3": W["c2"].replace(name="b3", B=2, T=333, M=10007, d=512, seed=14),
    # bf16 tensor-core projection with conv width 3 (unfused: CUDA-core gate/conv), d = 384
    "b4": W["c1"].replace(name="b4", B=3, T=150, K=2, D=64, d=384, w=3, dtype="bf16", seed=15),
    # fused passes with 128-channel tiles (d = 384 is not a multiple of 256), ragged rows
    "b5": W["c1"].replace(name="b5", B=2, T=237, K=4, D=64, d=384, w=4, dtype="bf16", seed=16),
}


@pytest.fixture(scope="module")
def eb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hashed_gram_embedding_02_b200 as eb
    return eb


def _run_forward(eb, ctx_obj, di, *, t_begin=0, state=None, add_residual=False, gamma=True):
    wl = di.wl
    y = di.empty_y()
    alpha = torch.empty(wl.n_tok, dtype=torch.float32, device=di.device)
    ctx_obj.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y, t_begin=t_begin,
                    gq=di.gq if gamma else None, gk=di.gk if gamma else None, conv_state=state,
                    alpha_out=alpha, add_residual=add_residual)
    torch.cuda.synchronize()
    return y, alpha


def _check_y(wl, y_gpu, y_ref, vt_win, cw):
    err = np.abs(y_gpu - y_ref)
    if wl.dtype == "f32":
        assert err.max() <= 1e-5, err.max()
    else:
        assert err.max() <= 2e-2, err.max()
        bound = bf16_bound(y_ref, vt_win, cw)
        bad = err > bound
        assert not bad.any(), (int(bad.sum()), float(err.max()), float((err - bound).max()))
    return float(err.max())


# ---------------------------------------------------------------- generators

def test_device_generators_match_host():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    inp = synth.Inputs(W["c2"])
    tab = inp.device_tables("cuda:0")
    rows = np.array([0, 1, 77, 999_999, 1_000_002])
    for j in (0, 5, 15):
        got = tab[j, torch.from_numpy(rows).cuda()].float().cpu().numpy()
        assert np.array_equal(got, inp.table_rows(j, rows))
    h = inp.device_hidden("cuda:0")
    sel = np.array([0, 5, 16383])
    assert np.array_equal(h[torch.from_numpy(sel).cuda()].float().cpu().numpy(), inp.hidden_rows(sel))


# ---------------------------------------------------------------- integer steps

@pytest.mark.parametrize("name", ["c1", "b2", "f2", "c2", "c3", "c4"])
def test_remap_and_hash_bitexact(eb, name):
    wl = SMALL.get(name) or W[name]
    inp = synth.Inputs(wl)
    ctx = eb.Engram(config_for(inp, eb))
    dev = "cuda:0"
    tok = torch.from_numpy(inp.tok).to(dev)
    P = torch.from_numpy(inp.P).to(dev)
    canon_ref, bad = oracle.remap(inp.tok, inp.P)
    assert bad == 0
    idx_ref, _ = oracle.hash_ids(canon_ref, wl.Vc, wl.orders, wl.K, inp.mult, inp.rows, wl.t_begin)

    canon = torch.empty_like(tok)
    eb.engram_remap(ctx.ctx, tok, tok.numel(), P, canon)
    idx_fused = torch.empty(wl.n_tok, wl.J, dtype=torch.int32, device=dev)
    eb.engram_hash(ctx.ctx, tok, P, wl.B, wl.T, wl.T, wl.t_begin, idx_fused)
    idx_canon = torch.empty_like(idx_fused)
    eb.engram_hash(ctx.ctx, canon, None, wl.B, wl.T, wl.T, wl.t_begin, idx_canon)
    torch.cuda.synchronize()
    assert np.array_equal(canon.cpu().numpy(), canon_ref)
    got = idx_fused.cpu().numpy().view(np.uint32)
    assert np.array_equal(got, idx_ref)
    assert np.array_equal(idx_canon.cpu().numpy().view(np.uint32), idx_ref)
    assert ctx.status() == (eb.ENGRAM_OK, 0)


def test_hash_strided_context_and_t_begin(eb):
    # ids laid out with a row stride larger than T; windows reach into [0, t_begin)
    wl = SMALL["b2"]
    inp = synth.Inputs(wl)
    ctx = eb.Engram(config_for(inp, eb))
    canon_ref, _ = oracle.remap(inp.tok, inp.P)
    for t_begin in (0, 1, 2, 5, wl.T - 1):
        ref, _ = oracle.hash_ids(canon_ref, wl.Vc, wl.orders, wl.K, inp.mult, inp.rows, t_begin)
        padded = np.zeros((wl.B, wl.T + 13), dtype=np.int32)
        padded[:, :wl.T] = inp.tok
        tok = torch.from_numpy(padded).cuda()
        P = torch.from_numpy(inp.P).cuda()
        idx = torch.empty(wl.B * (wl.T - t_begin), wl.J, dtype=torch.int32, device="cuda")
        eb.engram_hash(ctx.ctx, tok, P, wl.B, wl.T, wl.T + 13, t_begin, idx)
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy().view(np.uint32), ref), t_begin


def test_hash_extreme_primes(eb):
    """The device reduction of the 64-bit hash modulo each table size, at the
    smallest primes and at the largest allowed one (2^31 - 1), against the
    oracle's plain remainder, on ids drawn over the whole canonical range."""
    wl = W["c2"].replace(name="primes", B=3, T=2000, seed=41)
    inp = synth.Inputs(wl)
    rows = np.array([2, 3, 5, 2147483647, 2147483629, 1000003, 65521, 7919,
                     2, 3, 2147483647, 999983, 7, 11, 13, 2147483587], dtype=np.int64)
    assert all(synth._is_prime(int(r)) for r in rows)
    cfg = eb.make_config(orders=wl.orders, heads=wl.K, rows=[int(x) for x in rows], mult=inp.mult, row_dim=wl.D,
                         hidden=wl.d, conv_width=wl.w, vocab=wl.V, canon_vocab=wl.Vc, dtype=eb.ENGRAM_BF16)
    ctx = eb.Engram(cfg)
    rng = np.random.default_rng(5)
    inp.tok[:] = rng.integers(0, wl.V, size=inp.tok.shape)      # uniform ids: every bit of the products varies
    canon_ref, _ = oracle.remap(inp.tok, inp.P)
    ref, _ = oracle.hash_ids(canon_ref, wl.Vc, wl.orders, wl.K, inp.mult, rows.astype(np.uint32))
    idx = torch.empty(wl.n_tok, wl.J, dtype=torch.int32, device="cuda")
    eb.engram_hash(ctx.ctx, torch.from_numpy(inp.tok).cuda(), torch.from_numpy(inp.P).cuda(), wl.B, wl.T, wl.T, 0,
                   idx)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy().view(np.uint32), ref)


@pytest.mark.parametrize("name", ["c1", "b2", "c2"])
def test_gather_bitexact(eb, name):
    wl = SMALL.get(name) or W[name]
    inp = synth.Inputs(wl)
    ctx = eb.Engram(config_for(inp, eb))
    canon_ref, _ = oracle.remap(inp.tok, inp.P)
    idx_ref, _ = oracle.hash_ids(canon_ref, wl.Vc, wl.orders, wl.K, inp.mult, inp.rows, wl.t_begin)
    tables = inp.device_tables("cuda:0")
    idx = torch.from_numpy(idx_ref.view(np.int32)).cuda()
    e = torch.empty(wl.n_tok, wl.d_mem, dtype=tables.dtype, device="cuda")
    eb.engram_gather(ctx.ctx, idx, wl.n_tok, tables, e)
    torch.cuda.synchronize()
    if wl.n_tok * wl.d_mem <= 1 << 22:
        ref = oracle.gather(idx_ref, inp.rows, inp.all_tables())
        assert np.array_equal(e.float().cpu().numpy(), ref)
    else:
        pos = synth.sample_positions(wl, 512, seed=3)
        ref = oracle.gather_rows(idx_ref[pos], inp.rows, inp.table_rows)
        got = e[torch.from_numpy(pos).cuda()].float().cpu().numpy()
        assert np.array_equal(got, ref)


def test_gather_out_of_range_index_zero_row_and_flag(eb):
    wl = SMALL["b2"]
    inp = synth.Inputs(wl)
    ctx = eb.Engram(config_for(inp, eb))
    tables = inp.device_tables("cuda:0")
    idx_np = np.zeros((5, wl.J), dtype=np.uint32)
    idx_np[1, 2] = wl.M            # out of range: zero row + ENGRAM_ERR_INDEX
    idx_np[3, 0] = 0xFFFFFFFF      # invalid marker: zero row, no flag
    e = torch.full((5, wl.d_mem), 7.0, dtype=tables.dtype, device="cuda")
    eb.engram_gather(ctx.ctx, torch.from_numpy(idx_np.view(np.int32)).cuda(), 5, tables, e)
    st, flags = ctx.status()
    assert flags == eb.ENGRAM_ERR_INDEX and st == 7
    ref = oracle.gather(idx_np, inp.rows, inp.all_tables())
    assert np.array_equal(e.float().cpu().numpy(), ref)
    assert ctx.status() == (eb.ENGRAM_OK, 0)      # cleared by the read


# ---------------------------------------------------------------- whole forward

@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("add_residual", [False, True])
def test_forward_full_small(eb, name, add_residual):
    wl = SMALL[name]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    y, alpha = _run_forward(eb, ctx, di, add_residual=add_residual)
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    ref = oracle.forward_full(inp, add_residual=add_residual)
    np.testing.assert_allclose(to_np(alpha), ref.alpha, rtol=0, atol=2e-6)
    win = oracle.vt_windows(ref.vt, wl.B, wl.T - wl.t_begin, wl.w)
    _check_y(wl, to_np(y), ref.y, win, inp.conv_w)


@pytest.mark.parametrize("name", ["b3", "b5"])
@pytest.mark.parametrize("state", [False, True])
def test_forward_large_magnitude(eb, name, state):
    """Values far outside the test distribution: W_V scaled by 2^18 (|v~| and
    the tap sums beyond 65504, the fp16 range) and h by 2^6 with
    the residual.  Both scalings are powers of two, so the bf16 inputs stay
    exact and the oracle sees the same numbers.  Y must stay finite and within
    the relative bound (one bf16 rounding of Y plus the conv inputs' terms);
    an absolute 2e-2 has no meaning at these magnitudes."""
    wl = SMALL[name]
    inp = synth.Inputs(wl, gamma="random")
    inp.Wv = inp.Wv * np.float32(2.0 ** 18)
    di = DeviceInputs(inp)
    assert torch.equal(di.Wv.float().cpu(), torch.from_numpy(inp.Wv))
    di.h = di.h * 64.0
    h_host = inp.all_hidden() * 64.0
    hist = None
    st_dev = None
    if state:
        hist = inp.state_rows(np.arange(wl.B)) * 2.0 ** 14
        st_dev = torch.from_numpy(hist.astype(np.float32)).cuda().contiguous()
    ctx = eb.Engram(config_for(inp, eb))
    y, alpha = _run_forward(eb, ctx, di, add_residual=True, state=st_dev)
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    ref = oracle.forward_full(inp, add_residual=True, h=h_host, hist=hist)
    # beyond the fp16 range, both the gated values and the tap sums
    assert np.max(np.abs(ref.vt)) > 65504 and np.max(np.abs(ref.u)) > 65504
    win = oracle.vt_windows(ref.vt, wl.B, wl.T - wl.t_begin, wl.w, hist)
    yg = to_np(y)
    assert np.all(np.isfinite(yg))
    np.testing.assert_allclose(to_np(alpha), ref.alpha, rtol=0, atol=2e-6)
    err = np.abs(yg - ref.y)
    bound = bf16_bound(ref.y, win, inp.conv_w)
    bad = err > bound
    assert not bad.any(), (int(bad.sum()), float(err.max()), float((err - bound).max()))


@pytest.mark.parametrize("name", ["c2", "c3"])
def test_forward_full_size_sampled(eb, name):
    wl = W[name]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    y, alpha = _run_forward(eb, ctx, di, add_residual=True)
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    # every index, bit-exact
    canon_ref, _ = oracle.remap(inp.tok, inp.P)
    idx_ref, _ = oracle.hash_ids(canon_ref, wl.Vc, wl.orders, wl.K, inp.mult, inp.rows)
    idx = ctx.workspace[: wl.n_tok * wl.J * 4].view(torch.int32).view(wl.n_tok, wl.J)
    assert np.array_equal(idx.cpu().numpy().view(np.uint32), idx_ref)
    pos = synth.sample_positions(wl, 96, seed=5)
    ref = oracle.forward_rows(inp, pos, add_residual=True, idx=idx_ref)
    sel = torch.from_numpy(pos).cuda()
    np.testing.assert_allclose(to_np(alpha[sel]), ref.alpha, rtol=0, atol=2e-6)
    _check_y(wl, to_np(y[sel]), ref.y, ref.vt_win, inp.conv_w)


def _value_rows(wl, tiles=None):
    """Rows at the value pass's tile and warp boundaries.  With K >= 2048 the
    value pass runs contiguous tiles on CTA pairs (125 output rows per
    128-row CTA tile, starting 3 rows before), and the first three rows of
    warps 1-3 take their conv history from the previous warp's halo slot;
    otherwise tiles of four 29-row segments (116 rows).  `tiles`: the tile
    indices to cover (default all)."""
    contig = wl.d_mem >= 2048 and wl.dtype == "bf16"
    out, step = (125, 32) if contig else (116, 29)
    rows = set()
    n_tiles = (wl.n_tok + out - 1) // out
    for mt in (range(n_tiles) if tiles is None else [m % n_tiles for m in tiles]):
        base = mt * out - 3
        for q in range(4):
            for lane in ((3, 4) if q == 0 else ((0, 1, 2, 31) if contig else (3, 4))):
                r = base + step * q + lane
                if 0 <= r < wl.n_tok:
                    rows.add(r)
        if 0 <= base + 2 < wl.n_tok:
            rows.add(base + 2)
    return rows


# CTA-pair tiling (two CTAs per M = 256 MMA) engages once there are enough row
# tiles to occupy every SM pair; these shapes reach it with ragged ends: an odd
# number of value row tiles leaves the second CTA of the last pair without rows
PAIR_CASES = {
    "pair_a": W["c2"].replace(name="pair_a", B=2, T=2000, M=10007, seed=31),       # 4000 rows, 35 value tiles
    "pair_b": W["c2"].replace(name="pair_b", B=3, T=1501, M=10007, seed=32),       # 4503 rows, ragged 128-row band
    "pair_c": W["c2"].replace(name="pair_c", B=3, T=1376, M=10007, seed=33),       # 4128 rows, 33 key tiles (odd)
    # K = 2048: the value pass on contiguous pair tiles, 31 of them (the last
    # pair's second CTA holds no rows)
    "contig_a": W["c3"].replace(name="contig_a", B=2, T=1900, M=10007, seed=35),
}


@pytest.mark.parametrize("name", sorted(PAIR_CASES))
def test_cta_pair_tiling_sampled(eb, name):
    wl = PAIR_CASES[name]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    y, alpha = _run_forward(eb, ctx, di, add_residual=True)
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    # rows around every 128-row key band edge, the value pass's warp and tile
    # boundaries, the sequence ends, and random rows
    edges = set()
    for base in range(0, wl.n_tok, 128):
        for r in (base - 4, base - 1, base, base + 3):
            if 0 <= r < wl.n_tok:
                edges.add(r)
    edges |= _value_rows(wl, tiles=(0, 1, 2, 15, 16, -3, -2, -1))
    pos = np.array(sorted(edges | set(synth.sample_positions(wl, 64, seed=7).tolist())), dtype=np.int64)
    ref = oracle.forward_rows(inp, pos, add_residual=True)
    sel = torch.from_numpy(pos).cuda()
    np.testing.assert_allclose(to_np(alpha[sel]), ref.alpha, rtol=0, atol=2e-6)
    _check_y(wl, to_np(y[sel]), ref.y, ref.vt_win, inp.conv_w)


def test_decode_c4_with_state(eb):
    wl = W["c4"]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    state = inp.device_state("cuda:0").contiguous()
    hist = inp.state_rows(np.arange(wl.B))
    y, alpha = _run_forward(eb, ctx, di, t_begin=wl.t_begin, state=state)
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    pos = np.arange(wl.n_tok)
    ref = oracle.forward_rows(inp, pos, hist=hist)
    np.testing.assert_allclose(to_np(alpha), ref.alpha, rtol=0, atol=2e-6)
    _check_y(wl, to_np(y), ref.y, ref.vt_win, inp.conv_w)
    # the state now holds the last w-1 gated values: old rows 1..2, then the new one
    st = state.cpu().numpy()
    np.testing.assert_array_equal(st[:, :2], hist[:, 1:].astype(np.float32))
    vt_new = ref.vt_win[:, 0]
    assert np.max(np.abs(st[:, 2] - vt_new)) <= 2.0 ** -7 * np.max(np.abs(vt_new)) + 1e-6


@pytest.mark.parametrize("name", ["c1", "b1", "b2"])
def test_decode_after_prefill_matches_longer_prefill(eb, name):
    """Prefill T-1 positions with a conv state, then one decode step at t = T-1:
    the decode row equals the last row of a prefill over all T positions."""
    wl = SMALL[name]
    inp = synth.Inputs(wl)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    y_full, _ = _run_forward(eb, ctx, di)
    L = wl.T
    state = torch.zeros(wl.B, wl.w - 1, wl.d, dtype=torch.float32, device="cuda")
    # prefill of the first T-1 positions: tokens [B][T] with stride T, rows t < T-1
    tok_short = di.tok[:, : L - 1]
    h_rows = di.h.view(wl.B, L, wl.d)
    y1 = torch.empty(wl.B * (L - 1), wl.d, dtype=di.dtype, device="cuda")
    ctx.forward(tok_short, di.P, di.tables, h_rows[:, : L - 1].contiguous().view(-1, wl.d), di.Wk, di.Wv,
                di.conv_w, y1, gq=di.gq, gk=di.gk, conv_state=state)
    # decode step at t = T-1, n-gram context from the full token rows
    y2 = torch.empty(wl.B, wl.d, dtype=di.dtype, device="cuda")
    ctx.forward(di.tok, di.P, di.tables, h_rows[:, L - 1].contiguous(), di.Wk, di.Wv, di.conv_w, y2,
                t_begin=L - 1, gq=di.gq, gk=di.gk, conv_state=state)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    full = y_full.view(wl.B, L, wl.d)
    assert torch.equal(y1.view(wl.B, L - 1, wl.d), full[:, : L - 1])
    diff = (y2.float() - full[:, L - 1].float()).abs().max().item()
    # same v and alpha arithmetic on both paths; only a bf16 flip of v can differ
    assert diff <= (2e-2 if wl.dtype == "bf16" else 1e-6), diff


def test_invalid_token_flags_and_matches_oracle(eb):
    wl = SMALL["b1"]
    inp = synth.Inputs(wl)
    inp.tok[0, 17] = wl.V + 5        # outside the vocabulary
    inp.tok[1, 0] = -3
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    y, alpha = _run_forward(eb, ctx, di)
    st, flags = ctx.status()
    assert flags == eb.ENGRAM_ERR_TOKEN and st == 7
    ref = oracle.forward_full(inp)
    win = oracle.vt_windows(ref.vt, wl.B, wl.T, wl.w)
    _check_y(wl, to_np(y), ref.y, win, inp.conv_w)
    np.testing.assert_allclose(to_np(alpha), ref.alpha, rtol=0, atol=2e-6)


def test_forward_is_deterministic(eb):
    wl = SMALL["b3"]
    inp = synth.Inputs(wl)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    y1, a1 = _run_forward(eb, ctx, di)
    y2, a2 = _run_forward(eb, ctx, di)
    assert torch.equal(y1, y2) and torch.equal(a1, a2)


@pytest.mark.parametrize("name", ["b3", "pair_a"])
def test_dependent_launches_match_plain_launches(eb, name):
    """engram_forward launches the key pass as a programmatic dependent of the
    retrieval and the value pass as one of the key pass; with kernel timing
    on, events separate the kernels and the launches are plain.  Both must
    give the same bits.  A forward on other hidden states runs first, so a
    value epilogue that read alpha before the key pass completed would see
    different values."""
    wl = {**SMALL, **PAIR_CASES}[name]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    y0 = di.empty_y()
    ctx.forward(di.tok, di.P, di.tables, (di.h * 3).contiguous(), di.Wk, di.Wv, di.conv_w, y0, gq=di.gq, gk=di.gk,
                add_residual=True)
    y1, a1 = _run_forward(eb, ctx, di, add_residual=True)
    eb.engram_profile_enable(ctx.ctx, True)
    try:
        y2, a2 = _run_forward(eb, ctx, di, add_residual=True)
    finally:
        eb.engram_profile_enable(ctx.ctx, False)
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    assert torch.equal(y1, y2) and torch.equal(a1, a2)


@pytest.mark.parametrize("B,T,t_begin", [(1, 1, 0), (1, 2, 0), (2, 3, 1), (1, 129, 0), (5, 1, 0), (3, 4, 4)])
def test_edge_shapes(eb, B, T, t_begin):
    wl = SMALL["b1"].replace(B=B, T=T, t_begin=t_begin)
    inp = synth.Inputs(wl)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    if wl.n_tok == 0:
        y = torch.empty(0, wl.d, dtype=di.dtype, device="cuda")
        ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y, t_begin=t_begin)
        return
    y, _ = _run_forward(eb, ctx, di, t_begin=t_begin)
    ref = oracle.forward_full(inp)
    win = oracle.vt_windows(ref.vt, wl.B, wl.T - wl.t_begin, wl.w)
    _check_y(wl, to_np(y), ref.y, win, inp.conv_w)


def test_host_checks_launch_nothing(eb):
    from hashed_gram_embedding_02_b200 import binding
    wl = SMALL["b1"]
    inp = synth.Inputs(wl)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb), B=wl.B, L=wl.T)
    y = torch.full((wl.n_tok, wl.d), 3.0, dtype=di.dtype, device="cuda")
    # workspace one byte short
    with pytest.raises(binding.EngramError) as ei:
        eb.engram_forward(ctx.ctx, di.tok, wl.B, wl.T, wl.T, 0, di.P, di.tables, di.h, di.Wk, di.Wv, None, None,
                          di.conv_w, None, y, None, 0, ctx.workspace, ctx.workspace_bytes - 1)
    assert ei.value.status == binding.ENGRAM_E_NOMEM
    # misaligned output
    ybig = torch.zeros(wl.n_tok * wl.d + 8, dtype=di.dtype, device="cuda")
    with pytest.raises(binding.EngramError) as ei:
        eb.engram_forward(ctx.ctx, di.tok, wl.B, wl.T, wl.T, 0, di.P, di.tables, di.h, di.Wk, di.Wv, None, None,
                          di.conv_w, None, ybig[1:], None, 0, ctx.workspace, ctx.workspace_bytes)
    assert ei.value.status == binding.ENGRAM_E_INVAL
    # t_begin beyond T
    with pytest.raises(binding.EngramError):
        eb.engram_forward(ctx.ctx, di.tok, wl.B, wl.T, wl.T, wl.T + 1, di.P, di.tables, di.h, di.Wk, di.Wv, None,
                          None, di.conv_w, None, y, None, 0, ctx.workspace, ctx.workspace_bytes)
    torch.cuda.synchronize()
    assert bool((y == 3.0).all()) and bool((ybig == 0).all())


@pytest.mark.parametrize("name", ["b1", "b2", "b3", "c1"])
def test_project_v_and_partials(eb, name):
    """engram_project alone: v (storage dtype) and the per-group gate partials
    against the oracle's fp64 projections."""
    wl = SMALL[name]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    ref = oracle.forward_full(inp)
    e = torch.from_numpy(ref.e.astype(np.float32)).to(di.dtype).cuda()
    G = (wl.d + 127) // 128
    v = torch.empty(wl.n_tok, wl.d, dtype=torch.float32, device="cuda")
    part = torch.full((wl.n_tok, G, 4), float("nan"), dtype=torch.float32, device="cuda")
    eb.engram_project(ctx.ctx, e, wl.n_tok, di.h, di.Wk, di.Wv, di.gq, di.gk, v, part)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    vg = to_np(v)
    # fp32 accumulation of d_mem products: bounded by d_mem 2^-23 sum_q |e_q W_q|
    # (large relative to |v| only where the sum cancels)
    s_abs = np.abs(ref.e.astype(np.float64)) @ np.abs(inp.Wv.astype(np.float64)).T
    diff = np.abs(vg - ref.v)
    bound = wl.d_mem * 2.0 ** -23 * s_abs + 1e-30
    assert np.all(diff <= bound), float((diff / bound).max())
    if wl.dtype == "f32":
        assert diff.max() <= 1e-5
    h = inp.all_hidden()
    gg = inp.gq.astype(np.float64) * inp.gk.astype(np.float64)
    pg = part.cpu().numpy().astype(np.float64)
    for g in range(G):
        sl = slice(g * 128, min(wl.d, g * 128 + 128))
        want_qk = np.sum(gg[sl][None] * h[:, sl] * ref.k[:, sl], axis=1)
        want_kk = np.sum(ref.k[:, sl] ** 2, axis=1)
        want_hh = np.sum(h[:, sl].astype(np.float64) ** 2, axis=1)
        scale_qk = np.sum(np.abs(gg[sl][None] * h[:, sl] * ref.k[:, sl]), axis=1)
        np.testing.assert_allclose(pg[:, g, 0], want_qk, rtol=0, atol=1e-5 * (1 + scale_qk.max()))
        np.testing.assert_allclose(pg[:, g, 1], want_kk, rtol=2e-5, atol=1e-7)
        np.testing.assert_allclose(pg[:, g, 2], want_hh, rtol=2e-5, atol=1e-7)
        assert np.all(pg[:, g, 3] == 0)


@pytest.mark.parametrize("name", ["b1", "b3", "c1", "b2"])
def test_unfused_project_then_conv_matches_oracle(eb, name):
    """engram_project (v in fp32) followed by engram_conv, with a conv history:
    the standalone path gives the same result as the oracle."""
    wl = SMALL[name]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    hist = inp.state_rows(np.arange(wl.B))
    ref = oracle.forward_full(inp, add_residual=True, hist=hist)
    e = torch.from_numpy(ref.e.astype(np.float32)).to(di.dtype).cuda()
    G = (wl.d + 127) // 128
    v = torch.empty(wl.n_tok, wl.d, dtype=torch.float32, device="cuda")
    part = torch.empty(wl.n_tok, G, 4, dtype=torch.float32, device="cuda")
    eb.engram_project(ctx.ctx, e, wl.n_tok, di.h, di.Wk, di.Wv, di.gq, di.gk, v, part)
    state = torch.from_numpy(hist.astype(np.float32)).cuda()
    y = di.empty_y()
    alpha = torch.empty(wl.n_tok, dtype=torch.float32, device="cuda")
    eb.engram_conv(ctx.ctx, v, part, di.h, di.conv_w, wl.B, wl.T, state, y, alpha, 1)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    np.testing.assert_allclose(to_np(alpha), ref.alpha, rtol=0, atol=2e-6)
    win = oracle.vt_windows(ref.vt, wl.B, wl.T, wl.w, hist)
    _check_y(wl, to_np(y), ref.y, win, inp.conv_w)
    # new history = the last w-1 gated rows of every sequence
    want = ref.vt.reshape(wl.B, wl.T, wl.d)[:, wl.T - (wl.w - 1):]
    np.testing.assert_allclose(state.cpu().numpy(), want, rtol=0, atol=1e-5)


def test_pair_value_pass_with_history(eb):
    """A continued prefill on the contiguous pair tiles: each sequence's first
    three rows take their history from conv_state, rows at warp boundaries
    from the halo slots, and the last three rows become the new state."""
    wl = W["c3"].replace(name="pair_hist", B=2, T=2000, t_begin=100, M=10007, seed=34)
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    hist = inp.state_rows(np.arange(wl.B))
    state = inp.device_state("cuda:0").contiguous()
    L = wl.T - wl.t_begin
    y, alpha = _run_forward(eb, ctx, di, t_begin=wl.t_begin, state=state, add_residual=True)
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    rows = _value_rows(wl, tiles=(0, 1, 14, 15, 16, 29, 30))
    for b in range(wl.B):
        rows |= {b * L + t for t in (0, 1, 2, 3, L - 1)}
    pos = np.array(sorted(rows), dtype=np.int64)
    ref = oracle.forward_rows(inp, pos, add_residual=True, hist=hist)
    sel = torch.from_numpy(pos).cuda()
    np.testing.assert_allclose(to_np(alpha[sel]), ref.alpha, rtol=0, atol=2e-6)
    _check_y(wl, to_np(y[sel]), ref.y, ref.vt_win, inp.conv_w)
    last = oracle.forward_rows(inp, np.array([b * L + t for b in range(wl.B) for t in range(L - 3, L)]),
                               hist=hist)
    want = last.vt_win[:, 0].reshape(wl.B, 3, wl.d)
    vmax = float(np.abs(want).max())
    assert float(np.abs(state.cpu().numpy() - want).max()) <= 2.0 ** -10 * vmax + 1e-6


def test_pair_value_pass_short_sequences_with_history(eb):
    """1024 sequences of 4 new positions each (a decode-shaped call, L <= 8)
    at K = 2048: the value pass runs contiguous pair tiles and reads the conv
    history in the sequence-minor layout, and every row's history reaches
    into conv_state (the slow path), including rows at warp boundaries that
    otherwise take it from the halo slots."""
    wl = W["c3"].replace(name="ds_contig", B=1024, T=68, t_begin=64, M=10007, seed=36)
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    hist = inp.state_rows(np.arange(wl.B))
    state = inp.device_state("cuda:0").contiguous()
    L = wl.T - wl.t_begin
    y, alpha = _run_forward(eb, ctx, di, t_begin=wl.t_begin, state=state, add_residual=True)
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    rows = _value_rows(wl, tiles=(0, 1, 2, 16, 17, -2, -1))
    rows |= set(synth.sample_positions(wl, 48, seed=9).tolist())
    pos = np.array(sorted(rows), dtype=np.int64)
    ref = oracle.forward_rows(inp, pos, add_residual=True, hist=hist)
    sel = torch.from_numpy(pos).cuda()
    np.testing.assert_allclose(to_np(alpha[sel]), ref.alpha, rtol=0, atol=2e-6)
    _check_y(wl, to_np(y[sel]), ref.y, ref.vt_win, inp.conv_w)
    # the new history of a few sequences: their last three gated rows
    bs = np.array([0, 5, 511, 1023])
    last = oracle.forward_rows(inp, np.array([b * L + t for b in bs for t in range(L - 3, L)]), hist=hist)
    want = last.vt_win[:, 0].reshape(len(bs), 3, wl.d)
    got = state.cpu().numpy()[bs]
    assert float(np.abs(got - want).max()) <= 2.0 ** -10 * float(np.abs(want).max()) + 1e-6


@pytest.mark.parametrize("name", ["b1", "b3"])
def test_fused_prefill_with_history(eb, name):
    """Fused tensor-core path with a conv history at the start of every
    sequence (chunked prefill) and the history update."""
    wl = SMALL[name]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    hist = inp.state_rows(np.arange(wl.B))
    state = torch.from_numpy(hist.astype(np.float32)).cuda()
    y, alpha = _run_forward(eb, ctx, di, state=state, add_residual=True)
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    ref = oracle.forward_full(inp, add_residual=True, hist=hist)
    np.testing.assert_allclose(to_np(alpha), ref.alpha, rtol=0, atol=2e-6)
    win = oracle.vt_windows(ref.vt, wl.B, wl.T, wl.w, hist)
    _check_y(wl, to_np(y), ref.y, win, inp.conv_w)
    want = ref.vt.reshape(wl.B, wl.T, wl.d)[:, wl.T - (wl.w - 1):]
    np.testing.assert_allclose(state.cpu().numpy(), want, rtol=0, atol=1e-5)

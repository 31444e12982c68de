"""Training backward for the tables on the GPU against the oracle.

The distinct rows must match exactly (integers); each row's fp32 sum of k
gradient slices must lie within the bound of sequential fp32 summation,
(k - 1) * 2^-24 * sum |x| (Higham, Accuracy and Stability of Numerical
Algorithms, 2nd ed., section 4.2), plus one rounding of the result; the
result is the same on every run, bit for bit."""

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import config_for

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
CASES = {
    "g1": W["c1"].replace(name="g1", B=3, T=200, K=4, D=64, d=256, dtype="bf16", seed=71),
    "g2": W["c1"].replace(name="g2", B=2, T=100, seed=72),                      # fp32 tables
    "c3": W["c3"],
}


@pytest.fixture(scope="module")
def eb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hashed_gram_embedding_02_b200 as eb
    return eb


def _idx(eb, ctx, inp):
    wl = inp.wl
    idx = torch.empty(wl.n_tok, wl.J, dtype=torch.int32, device="cuda")
    eb.engram_hash(ctx.ctx, torch.from_numpy(inp.tok).cuda(), torch.from_numpy(inp.P).cuda(), wl.B, wl.T, wl.T,
                   wl.t_begin, idx)
    return idx


def _de(wl, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    return (torch.randn(wl.n_tok, wl.d_mem, device="cuda", generator=g) * 0.01).to(dt)


def _sorted(rows, grad):
    r = rows.cpu().numpy().astype(np.int64)
    order = np.argsort(r)
    return r[order], grad.cpu().numpy()[order]


def _check(inp, idx_np, de_np, rows, grad):
    wl = inp.wl
    keys, ref = oracle.table_grad(idx_np, inp.rows, de_np, wl.D)
    _, absum = oracle.table_grad(idx_np, inp.rows, np.abs(de_np), wl.D)
    _, cnt = oracle.table_grad(idx_np, inp.rows, np.ones_like(de_np), wl.D)
    r, g = _sorted(rows, grad)
    assert np.array_equal(r, keys)
    bound = np.maximum(cnt - 1, 0) * 2.0 ** -24 * absum + 2.0 ** -24 * np.abs(ref) + 1e-38
    err = np.abs(g - ref)
    assert not (err > bound).any(), (int((err > bound).sum()), float(err.max()))


@pytest.mark.parametrize("name", sorted(CASES))
def test_table_grad_matches_oracle_and_is_deterministic(eb, name):
    wl = CASES[name]
    inp = synth.Inputs(wl)
    ctx = eb.Engram(config_for(inp, eb))
    idx = _idx(eb, ctx, inp)
    de = _de(wl, 5)
    rows, grad, _ = ctx.table_grad(idx, de)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    idx_np = idx.cpu().numpy().view(np.uint32)
    _check(inp, idx_np, de.float().cpu().numpy().astype(np.float64), rows, grad)
    rows2, grad2, _ = ctx.table_grad(idx, de)
    r1, g1 = _sorted(rows, grad)
    r2, g2 = _sorted(rows2, grad2)
    assert np.array_equal(r1, r2) and np.array_equal(g1, g2)


def test_table_grad_skips_invalid_lookups(eb):
    wl = CASES["g1"]
    inp = synth.Inputs(wl)
    inp.tok[0, 10] = wl.V + 3
    ctx = eb.Engram(config_for(inp, eb))
    idx = _idx(eb, ctx, inp)
    idx_np = idx.cpu().numpy().view(np.uint32)
    assert (idx_np == 0xFFFFFFFF).sum() > 0
    de = _de(wl, 6)
    rows, grad, _ = ctx.table_grad(idx, de)
    torch.cuda.synchronize()
    ctx.status()                                   # clears the token flag
    _check(inp, idx_np, de.float().cpu().numpy().astype(np.float64), rows, grad)


def test_table_grad_one_row_looked_up_everywhere(eb):
    """A degenerate batch: one token repeated, so every lookup of a table hits
    the same row (segments of n_tok lookups)."""
    wl = CASES["g1"].replace(name="g3", B=1, T=2048)
    inp = synth.Inputs(wl)
    inp.tok[:] = 7
    ctx = eb.Engram(config_for(inp, eb))
    idx = _idx(eb, ctx, inp)
    de = _de(wl, 7)
    rows, grad, _ = ctx.table_grad(idx, de)
    torch.cuda.synchronize()
    idx_np = idx.cpu().numpy().view(np.uint32)
    _check(inp, idx_np, de.float().cpu().numpy().astype(np.float64), rows, grad)
    assert len(rows) <= 3 * wl.J          # the PAD windows at the start, then one n-gram per order


@pytest.mark.parametrize("name", ["g1", "g2"])
def test_table_sgd_updates_exactly_the_touched_rows(eb, name):
    wl = CASES[name]
    inp = synth.Inputs(wl)
    ctx = eb.Engram(config_for(inp, eb))
    tables = inp.device_tables("cuda:0")
    before = tables.clone()
    idx = _idx(eb, ctx, inp)
    de = _de(wl, 8)
    rows, grad, cnt = ctx.table_grad(idx, de)
    lr = 0.5
    eb.engram_table_sgd(ctx.ctx, rows, grad, cnt, rows.numel(), tables, lr)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    flat_b = before.reshape(-1, wl.D).float().cpu().numpy().astype(np.float64)
    flat_a = tables.reshape(-1, wl.D).float().cpu().numpy().astype(np.float64)
    r, g = _sorted(rows, grad)
    want = flat_b[r] - lr * g.astype(np.float64)
    # one rounding to the table dtype (fp32 arithmetic first): within one unit in the last place
    ulp = np.spacing(np.abs(want).astype(np.float32)).astype(np.float64) * (65536.0 if wl.dtype == "bf16" else 1.0)
    assert np.all(np.abs(flat_a[r] - want) <= ulp + 1e-30)
    untouched = np.setdiff1d(np.arange(flat_b.shape[0]), r)
    assert np.array_equal(flat_a[untouched], flat_b[untouched])

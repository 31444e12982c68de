"""Failure detection in the tensor-core passes, without a GPU fault.

Every mbarrier wait in the projection kernels is bounded (about 2 s).  The
test hook engram_debug_stall_next makes CTA 0 of the next key pass announce
the bytes of its first operand stage and never load them, so the MMA warp's
wait on that stage runs out.  The kernel must then flag ENGRAM_ERR_TIMEOUT,
drain what it issued and return; the host reads ENGRAM_E_TIMEOUT, and the
same context computes the next forward correctly.  Covered on the single-CTA
key pass and on the CTA-pair key pass (cluster of two, which also has to
stop its peer and leave together)."""

import time

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import DeviceInputs, bf16_bound, config_for, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
CASES = {
    # 666 rows: single-CTA key pass
    "single": W["c2"].replace(name="single", B=2, T=333, M=10007, d=512, seed=51),
    # 4000 rows x 10 channel tiles: CTA-pair key pass
    "pair": W["c2"].replace(name="pair", B=2, T=2000, M=10007, seed=52),
}


@pytest.fixture(scope="module")
def eb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hashed_gram_embedding_02_b200 as eb
    return eb


@pytest.mark.parametrize("name", sorted(CASES))
def test_stalled_wait_times_out_and_context_recovers(eb, name):
    wl = CASES[name]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    y = di.empty_y()
    eb.engram_debug_stall_next(ctx.ctx)
    t0 = time.time()
    ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y, gq=di.gq, gk=di.gk, add_residual=True)
    st, flags = ctx.status()                      # synchronises the stream
    elapsed = time.time() - t0
    assert st == eb.ENGRAM_E_TIMEOUT and flags & eb.ENGRAM_ERR_TIMEOUT, (st, flags)
    assert elapsed < 30.0                         # every wait, the drain's included, is bounded
    assert ctx.status() == (eb.ENGRAM_OK, 0)     # read and cleared

    # the same context and workspace give the right answer next time
    y2 = di.empty_y()
    alpha = torch.empty(wl.n_tok, dtype=torch.float32, device="cuda")
    ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y2, gq=di.gq, gk=di.gk, alpha_out=alpha,
                add_residual=True)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    pos = synth.sample_positions(wl, 64, seed=11)
    ref = oracle.forward_rows(inp, pos, add_residual=True)
    sel = torch.from_numpy(pos).cuda()
    np.testing.assert_allclose(to_np(alpha[sel]), ref.alpha, rtol=0, atol=2e-6)
    err = np.abs(to_np(y2[sel]) - ref.y)
    assert err.max() <= 2e-2
    assert not (err > bf16_bound(ref.y, ref.vt_win, inp.conv_w)).any()


def test_decode_stalled_wait_times_out_and_context_recovers(eb):
    """The same on the decode key pass (clusters of four CTAs splitting K): the
    stalled CTA votes to abort, its cluster skips the partial exchange, and
    every CTA still meets the cluster barriers and leaves."""
    wl = W["c2"].replace(name="decode", B=64, T=4, t_begin=3, M=10007, seed=53)
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    state = inp.device_state("cuda:0").contiguous()
    y = di.empty_y()
    eb.engram_debug_stall_next(ctx.ctx)
    t0 = time.time()
    ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y, t_begin=wl.t_begin, gq=di.gq, gk=di.gk,
                conv_state=state.clone(), add_residual=True)
    st, flags = ctx.status()
    elapsed = time.time() - t0
    assert st == eb.ENGRAM_E_TIMEOUT and flags & eb.ENGRAM_ERR_TIMEOUT, (st, flags)
    assert elapsed < 30.0
    assert ctx.status() == (eb.ENGRAM_OK, 0)

    y2 = di.empty_y()
    alpha = torch.empty(wl.n_tok, dtype=torch.float32, device="cuda")
    ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y2, t_begin=wl.t_begin, gq=di.gq, gk=di.gk,
                conv_state=state, alpha_out=alpha, add_residual=True)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    hist = inp.state_rows(np.arange(wl.B))
    ref = oracle.forward_rows(inp, np.arange(wl.n_tok), add_residual=True, hist=hist)
    np.testing.assert_allclose(to_np(alpha), ref.alpha, rtol=0, atol=2e-6)
    err = np.abs(to_np(y2) - ref.y)
    assert err.max() <= 2e-2
    assert not (err > bf16_bound(ref.y, ref.vt_win, inp.conv_w)).any()

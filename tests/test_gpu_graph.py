"""engram_forward and engram_forward_host captured into a CUDA graph: a replay
gives the same bits as an eager call, for a prefill and for a decode step
(whose conv state the replay updates in place, as the eager call does); the
host-buffer call's copies replay from and to the same pinned buffers."""

import numpy as np
import pytest

import synth
from gpu_helpers import DeviceInputs, config_for

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
CASES = {
    "prefill": W["c2"].replace(name="prefill", B=2, T=333, M=10007, d=512, seed=71),
    "decode": W["c4"].replace(name="decode", M=10007, T=16, t_begin=15, seed=72),
}


@pytest.fixture(scope="module")
def eb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hashed_gram_embedding_02_b200 as eb
    return eb


@pytest.mark.parametrize("name", sorted(CASES))
def test_graph_replay_matches_eager(eb, name):
    wl = CASES[name]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb), B=wl.B, L=wl.T - wl.t_begin)
    s0 = inp.device_state("cuda:0").contiguous() if wl.t_begin > 0 else None
    y = di.empty_y()
    alpha = torch.empty(wl.n_tok, dtype=torch.float32, device="cuda")
    state = s0.clone() if s0 is not None else None

    def step():
        ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y, t_begin=wl.t_begin, gq=di.gq,
                    gk=di.gk, conv_state=state, alpha_out=alpha, add_residual=True)

    step()
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    y_eager, a_eager = y.clone(), alpha.clone()
    st_eager = state.clone() if state is not None else None

    g = torch.cuda.CUDAGraph()
    if state is not None:
        state.copy_(s0)
    with torch.cuda.graph(g):
        step()
    # capture records the launches without running them
    if state is not None:
        state.copy_(s0)
    y.zero_()
    alpha.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    assert torch.equal(y, y_eager) and torch.equal(alpha, a_eager)
    if state is not None:
        assert torch.equal(state, st_eager)
    # a second replay from the same starting state: the same bits again
    if state is not None:
        state.copy_(s0)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, y_eager)


def test_profile_events_inside_a_graph(eb):
    """With kernel timing on, a captured forward records its events as graph
    nodes: every replay yields positive per-kernel durations, and a failed
    read leaves no pending error behind for the next launch."""
    wl = CASES["decode"]
    inp = synth.Inputs(wl)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb), B=wl.B, L=1)
    state = inp.device_state("cuda:0").contiguous()
    y = di.empty_y()

    def step():
        ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y, t_begin=wl.t_begin, gq=di.gq,
                    gk=di.gk, conv_state=state, add_residual=True)

    step()
    eb.engram_profile_enable(ctx.ctx, True)
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        for _ in range(3):
            g.replay()
            torch.cuda.synchronize()
            prof = eb.engram_profile_read(ctx.ctx)
            assert [n for n, _ in prof] == ["retrieve", "gate_kv_decode", "conv_decode"], prof
            assert all(t > 0.0 for _, t in prof), prof
        del g
    finally:
        eb.engram_profile_enable(ctx.ctx, False)
    step()                                   # an eager call after the graph
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)


@pytest.mark.parametrize("name,chunk_rows", [("prefill", 0), ("prefill", 50), ("decode", 0)])
def test_host_forward_graph_replay_matches_eager(eb, name, chunk_rows):
    wl = CASES[name]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb), B=wl.B, L=wl.T - wl.t_begin)
    s0 = inp.device_state("cuda:0").contiguous() if wl.t_begin > 0 else None
    state = s0.clone() if s0 is not None else None
    tok_h = di.tok.cpu().contiguous().pin_memory()
    h_h = di.h.cpu().contiguous().pin_memory()
    y_h = torch.empty(wl.n_tok, wl.d, dtype=di.dtype).pin_memory()

    def step():
        ctx.forward_host(tok_h, di.P, di.tables, h_h, di.Wk, di.Wv, di.conv_w, y_h, t_begin=wl.t_begin, gq=di.gq,
                         gk=di.gk, conv_state=state, add_residual=True, chunk_rows=chunk_rows)

    step()
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    y_eager = y_h.clone()
    st_eager = state.clone() if state is not None else None
    g = torch.cuda.CUDAGraph()
    if state is not None:
        state.copy_(s0)
    with torch.cuda.graph(g):
        step()
    torch.cuda.synchronize()
    for _ in range(2):
        if state is not None:
            state.copy_(s0)
        y_h.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert ctx.status() == (eb.ENGRAM_OK, 0)
        assert torch.equal(y_h, y_eager)
        if state is not None:
            assert torch.equal(state, st_eager)
    del g

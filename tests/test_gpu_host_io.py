"""engram_forward_host: the forward with ids, hidden states and output in host
memory, pipelined in chunks of positions over PCIe.  Its output must match the
oracle as the device-buffer forward does, for every chunk size (the conv
history crosses chunk boundaries through the carried state), with pinned and
with pageable host buffers, in prefill, in a continued prefill (t_begin > 0)
and in decode."""

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import DeviceInputs, bf16_bound, config_for, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
# bf16 fused tensor-core path with ragged row tiles; fp32 CUDA-core path
B3 = W["c2"].replace(name="b3", B=2, T=333, M=10007, d=512, seed=14)
C1 = W["c1"]


@pytest.fixture(scope="module")
def eb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hashed_gram_embedding_02_b200 as eb
    return eb


def _check(wl, y, ref_y, win, cw):
    err = np.abs(y - ref_y)
    if wl.dtype == "f32":
        assert err.max() <= 1e-5, err.max()
        return
    assert err.max() <= 2e-2, err.max()
    bad = err > bf16_bound(ref_y, win, cw)
    assert not bad.any(), int(bad.sum())


def _host(t, pin):
    t = t.cpu().contiguous()
    return t.pin_memory() if pin else t


@pytest.mark.parametrize("wl", [B3, C1], ids=["b3", "c1"])
@pytest.mark.parametrize("chunk_rows", [0, 1, 7, 116, 1000])
def test_host_forward_matches_oracle(eb, wl, chunk_rows):
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    tok_h = _host(di.tok, True)
    h_h = _host(di.h, True)
    y_h = torch.full((wl.n_tok, wl.d), float("nan"), dtype=di.dtype).pin_memory()
    ctx.forward_host(tok_h, di.P, di.tables, h_h, di.Wk, di.Wv, di.conv_w, y_h, gq=di.gq, gk=di.gk,
                     add_residual=True, chunk_rows=chunk_rows)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    ref = oracle.forward_full(inp, add_residual=True)
    win = oracle.vt_windows(ref.vt, wl.B, wl.T, wl.w)
    _check(wl, y_h.double().numpy(), ref.y, win, inp.conv_w)


def test_host_forward_ramped_chunks_match_oracle(eb):
    """A batch long enough for the default schedule's ramp (16 sequences of
    1000 positions, d = 2560: 16 MiB middle chunks of 204 positions, ends of
    25, 51 and 102): rows at and next to every chunk boundary match the
    oracle, and the workspace is the one of 204-position chunks."""
    wl = W["c2"].replace(name="ramp", B=16, T=1000, M=10007, seed=15)
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    assert (eb.engram_host_workspace_bytes(ctx.ctx, wl.B, wl.T, 0, 0)
            == eb.engram_host_workspace_bytes(ctx.ctx, wl.B, wl.T, 0, 204))
    y_h = torch.full((wl.n_tok, wl.d), float("nan"), dtype=di.dtype).pin_memory()
    ctx.forward_host(_host(di.tok, True), di.P, di.tables, _host(di.h, True), di.Wk, di.Wv, di.conv_w, y_h,
                     gq=di.gq, gk=di.gk, add_residual=True)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    assert not torch.isnan(y_h.float()).any()
    bounds = [0, 25, 76, 178, 382, 586, 790, 822, 924, 975]
    ts = sorted({t for b0 in bounds for t in (b0 - 1, b0, b0 + 1, b0 + 2, b0 + 3) if 0 <= t < wl.T})
    pos = np.array([b * wl.T + t for b in (0, 7, 15) for t in ts], dtype=np.int64)
    ref = oracle.forward_rows(inp, pos, add_residual=True)
    _check(wl, y_h[torch.from_numpy(pos)].double().numpy(), ref.y, ref.vt_win, inp.conv_w)


def test_host_forward_pageable_equals_pinned(eb):
    wl = B3
    inp = synth.Inputs(wl)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    out = []
    for pin in (True, False):
        y_h = _host(torch.zeros(wl.n_tok, wl.d, dtype=di.dtype), pin)
        ctx.forward_host(_host(di.tok, pin), di.P, di.tables, _host(di.h, pin), di.Wk, di.Wv, di.conv_w, y_h,
                         chunk_rows=50)
        torch.cuda.synchronize()
        out.append(y_h.clone())
    assert torch.equal(out[0], out[1])


def test_host_forward_equals_device_forward_in_one_chunk(eb):
    """One chunk (no carried history) runs exactly the device forward's kernels."""
    wl = B3
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    y_d = di.empty_y()
    ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y_d, gq=di.gq, gk=di.gk, add_residual=True)
    y_h = torch.empty(wl.n_tok, wl.d, dtype=di.dtype).pin_memory()
    ctx.forward_host(_host(di.tok, True), di.P, di.tables, _host(di.h, True), di.Wk, di.Wv, di.conv_w, y_h,
                     gq=di.gq, gk=di.gk, add_residual=True, chunk_rows=wl.T)
    torch.cuda.synchronize()
    assert torch.equal(y_h, y_d.cpu())


@pytest.mark.parametrize("chunk_rows", [0, 13])
def test_host_forward_continued_prefill_with_state(eb, chunk_rows):
    """t_begin > 0 with a caller history: only the id window from t_begin - 2
    is copied, the history carries through the chunks, and the final state is
    the one the device forward leaves."""
    wl = B3.replace(t_begin=120)
    inp = synth.Inputs(wl)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    hist = inp.state_rows(np.arange(wl.B))
    state0 = inp.device_state("cuda:0").contiguous()
    s_dev = state0.clone()
    y_d = di.empty_y()
    ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y_d, t_begin=wl.t_begin, conv_state=s_dev)
    s_host = state0.clone()
    y_h = torch.empty(wl.n_tok, wl.d, dtype=di.dtype).pin_memory()
    ctx.forward_host(_host(di.tok, True), di.P, di.tables, _host(di.h, True), di.Wk, di.Wv, di.conv_w, y_h,
                     t_begin=wl.t_begin, conv_state=s_host, chunk_rows=chunk_rows)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    ref = oracle.forward_full(inp, hist=hist)
    win = oracle.vt_windows(ref.vt, wl.B, wl.T - wl.t_begin, wl.w, hist=hist)
    _check(wl, y_h.double().numpy(), ref.y, win, inp.conv_w)
    vmax = float(np.abs(ref.vt).max())
    assert float((s_host - s_dev).abs().max()) <= 2.0 ** -10 * vmax + 1e-6


def test_host_forward_decode_c4_shape(eb):
    """Decode at the c4 shape (256 sequences of 8192 ids, one new position
    each): the copies carry 3 ids per sequence, not the whole context."""
    wl = W["c4"]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    state0 = inp.device_state("cuda:0").contiguous()
    s_dev, s_host = state0.clone(), state0.clone()
    y_d = di.empty_y()
    ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y_d, t_begin=wl.t_begin, gq=di.gq, gk=di.gk,
                conv_state=s_dev)
    y_h = torch.empty(wl.n_tok, wl.d, dtype=di.dtype).pin_memory()
    ctx.forward_host(_host(di.tok, True), di.P, di.tables, _host(di.h, True), di.Wk, di.Wv, di.conv_w, y_h,
                     t_begin=wl.t_begin, gq=di.gq, gk=di.gk, conv_state=s_host)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    assert torch.equal(y_h, y_d.cpu())
    assert torch.equal(s_host, s_dev)
    # scratch beyond one forward's and the four h/Y chunk buffers: the id window only
    extra = (eb.engram_host_workspace_bytes(ctx.ctx, wl.B, wl.T, wl.t_begin, 0)
             - eb.engram_workspace_bytes(ctx.ctx, wl.B, 1) - 4 * wl.B * wl.d * 2)
    assert 0 < extra < 64 << 10

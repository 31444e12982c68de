"""Multi-branch Engram on the GPU against the oracle, through the C ABI.

M branches share the tables, W_V and the conv taps; each has its own W_K,
RMSNorm gains, hidden state, gate, conv history and output.  The key pass
runs one GEMM over the stacked W_K^(1..M) and the value pass computes v once
for all branches.  Gates within 2e-6; Y within 2e-2 and the elementwise
bf16 bound; M = 1 equals engram_forward bit for bit."""

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import DeviceInputs, bf16_bound, config_for, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
CASES = {
    # 256-channel tiles, several row tiles, ragged tail
    "m1": W["c2"].replace(name="m1", B=2, T=333, M=10007, d=512, seed=61),
    # 128-channel tiles (d = 384)
    "m2": W["c1"].replace(name="m2", B=3, T=150, K=4, D=64, d=384, w=4, dtype="bf16", seed=62),
}


@pytest.fixture(scope="module")
def eb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hashed_gram_embedding_02_b200 as eb
    return eb


def _device_branches(branches, device="cuda:0"):
    h = torch.stack([b.device_hidden(device) for b in branches]).contiguous()
    Wk = torch.stack([torch.from_numpy(b.Wk).to(torch.bfloat16) for b in branches]).to(device).contiguous()
    gq = torch.stack([torch.from_numpy(b.gq) for b in branches]).to(device).contiguous()
    gk = torch.stack([torch.from_numpy(b.gk) for b in branches]).to(device).contiguous()
    return h, Wk, gq, gk


def _check(wl, y, ref_y, vt, cw, hist=None):
    L = wl.T - wl.t_begin
    for m in range(y.shape[0]):
        win = oracle.vt_windows(vt[m], wl.B, L, wl.w, None if hist is None else hist[m])
        err = np.abs(to_np(y[m]) - ref_y[m])
        assert err.max() <= 2e-2, (m, err.max())
        bad = err > bf16_bound(ref_y[m], win, cw)
        assert not bad.any(), (m, int(bad.sum()))


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("M", [1, 2, 4])
def test_multibranch_matches_oracle(eb, name, M):
    wl = CASES[name]
    inp = synth.Inputs(wl, gamma="random")
    branches = [synth.branch_inputs(inp, m) for m in range(M)]
    di = DeviceInputs(inp)
    h, Wk, gq, gk = _device_branches(branches)
    ctx = eb.Engram(config_for(inp, eb))
    y = torch.full((M, wl.n_tok, wl.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    alpha = torch.empty(M, wl.n_tok, dtype=torch.float32, device="cuda")
    ctx.forward_multibranch(di.tok, di.P, di.tables, h, Wk, di.Wv, di.conv_w, y, gq=gq, gk=gk, alpha_out=alpha,
                            add_residual=True)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    ref = oracle.forward_multibranch(branches, add_residual=True)
    np.testing.assert_allclose(to_np(alpha), ref.alpha, rtol=0, atol=2e-6)
    _check(wl, y, ref.y, ref.vt, inp.conv_w)
    if M == 1:
        y1 = di.empty_y()
        ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y1, gq=di.gq, gk=di.gk, add_residual=True)
        torch.cuda.synchronize()
        assert torch.equal(y1, y[0])


@pytest.mark.parametrize("decode", [False, True])
def test_multibranch_with_conv_history(eb, decode):
    """Per-branch histories in and out: prefill with a history, and a decode
    step (one position per sequence, the sequence-minor history layout)."""
    M = 3
    wl = CASES["m1"].replace(name="mh", B=4, T=40, t_begin=39 if decode else 0, seed=63)
    inp = synth.Inputs(wl, gamma="random")
    branches = [synth.branch_inputs(inp, m) for m in range(M)]
    di = DeviceInputs(inp)
    h, Wk, gq, gk = _device_branches(branches)
    hist = np.stack([b.state_rows(np.arange(wl.B)) for b in branches])
    state = torch.from_numpy(hist.astype(np.float32)).cuda().contiguous()
    ctx = eb.Engram(config_for(inp, eb))
    y = torch.empty(M, wl.n_tok, wl.d, dtype=torch.bfloat16, device="cuda")
    alpha = torch.empty(M, wl.n_tok, dtype=torch.float32, device="cuda")
    ctx.forward_multibranch(di.tok, di.P, di.tables, h, Wk, di.Wv, di.conv_w, y, t_begin=wl.t_begin, gq=gq, gk=gk,
                            conv_state=state, alpha_out=alpha)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    ref = oracle.forward_multibranch(branches, hist=hist)
    np.testing.assert_allclose(to_np(alpha), ref.alpha, rtol=0, atol=2e-6)
    _check(wl, y, ref.y, ref.vt, inp.conv_w, hist)
    # each branch's new history: its last w-1 gated values (within the extended sequence)
    L = wl.T - wl.t_begin
    st = state.cpu().numpy()
    for m in range(M):
        ext = np.concatenate([hist[m], ref.vt[m].reshape(wl.B, L, wl.d)], axis=1)
        want = ext[:, -(wl.w - 1):]
        assert np.max(np.abs(st[m] - want)) <= 2.0 ** -7 * np.max(np.abs(want)) + 1e-6, m


def test_multibranch_full_size_c3_sampled(eb):
    """c3 with four branches: every index, and the gates and Y of every branch
    at sampled rows (the oracle evaluates them one by one)."""
    import types
    M = 4
    wl = W["c3"]
    inp = synth.Inputs(wl, gamma="random")
    branches = [synth.branch_inputs(inp, m) for m in range(M)]
    di = DeviceInputs(inp)
    h, Wk, gq, gk = _device_branches(branches)
    del di.h
    ctx = eb.Engram(config_for(inp, eb))
    y = torch.empty(M, wl.n_tok, wl.d, dtype=torch.bfloat16, device="cuda")
    alpha = torch.empty(M, wl.n_tok, dtype=torch.float32, device="cuda")
    ctx.forward_multibranch(di.tok, di.P, di.tables, h, Wk, di.Wv, di.conv_w, y, gq=gq, gk=gk, alpha_out=alpha,
                            add_residual=True)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    canon, _ = oracle.remap(inp.tok, inp.P)
    idx_ref, _ = oracle.hash_ids(canon, wl.Vc, wl.orders, wl.K, inp.mult, inp.rows)
    idx = ctx.mb_workspace[: wl.n_tok * wl.J * 4].view(torch.int32).view(wl.n_tok, wl.J)
    assert np.array_equal(idx.cpu().numpy().view(np.uint32), idx_ref)
    pos = synth.sample_positions(wl, 64, seed=9)
    sel = torch.from_numpy(pos).cuda()
    for m in range(M):
        br = branches[m]
        one = types.SimpleNamespace(wl=wl, tok=inp.tok, P=inp.P, mult=inp.mult, rows=inp.rows, Wv=inp.Wv,
                                    conv_w=inp.conv_w, Wk=br.Wk, gq=br.gq, gk=br.gk, hidden_rows=br.hidden_rows,
                                    table_rows=inp.table_rows)
        ref = oracle.forward_rows(one, pos, add_residual=True, idx=idx_ref)
        np.testing.assert_allclose(to_np(alpha[m][sel]), ref.alpha, rtol=0, atol=2e-6)
        err = np.abs(to_np(y[m][sel]) - ref.y)
        assert err.max() <= 2e-2, (m, err.max())
        assert not (err > bf16_bound(ref.y, ref.vt_win, inp.conv_w)).any(), m


def test_multibranch_rejects_unsupported(eb):
    wl = W["c1"]          # fp32: no tensor-core path
    inp = synth.Inputs(wl)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    y = torch.empty(2, wl.n_tok, wl.d, device="cuda")
    h = torch.stack([di.h, di.h])
    Wk = torch.stack([di.Wk, di.Wk])
    with pytest.raises(eb.EngramError) as err:
        ctx.forward_multibranch(di.tok, di.P, di.tables, h, Wk, di.Wv, di.conv_w, y)
    assert err.value.status == eb.ENGRAM_E_UNSUPPORTED

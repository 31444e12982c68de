"""The FP8 (E4M3) path against the oracle: tables, e, W_K and W_V as E4M3
codes, the projections as tcgen05 kind::f8f6f4 GEMMs with fp32 accumulation
and per-channel dequantisation, h and Y in bf16.

The oracle computes on the decoded values (the decoding pinned to the E4M3
definition in test_oracle_pins.py), so the comparison covers the GEMMs, the
scales, the gate and the conv: gates within 2e-6, Y within 2e-2 and the
elementwise bf16 bound."""

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import DeviceInputs, bf16_bound, config_for, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
CASES = {
    # d_mem 512, 256-channel tiles, ragged rows
    "f8a": W["c1"].replace(name="f8a", B=2, T=237, K=4, D=64, d=256, dtype="fp8", seed=81),
    # d_mem 1024 (c2's rows), 128-channel tiles (d = 384)
    "f8b": W["c2"].replace(name="f8b", B=2, T=150, M=10007, d=384, dtype="fp8", seed=82),
}


@pytest.fixture(scope="module")
def eb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hashed_gram_embedding_02_b200 as eb
    return eb


def _branches_dev(branches, device="cuda:0"):
    dd = [b.device_dense(device) for b in branches]
    h = torch.stack([b.device_hidden(device) for b in branches]).contiguous()
    Wk = torch.stack([d["Wk"] for d in dd]).contiguous()
    ks = torch.stack([d["k_scale"] for d in dd]).contiguous()
    gq = torch.stack([d["gq"] for d in dd]).contiguous()
    gk = torch.stack([d["gk"] for d in dd]).contiguous()
    return h, Wk, ks, gq, gk


def test_device_codes_decode_to_the_host_values(eb):
    """The E4M3 codes the device holds decode (oracle definition) to the
    values the oracle computes with, tables and weights."""
    wl = CASES["f8b"]
    inp = synth.Inputs(wl)
    tab = inp.device_tables("cuda:0")
    assert tab.dtype == torch.uint8
    rows = np.array([0, 1, 77, wl.M - 1])
    for j in (0, 7, 15):
        codes = tab[j, torch.from_numpy(rows).cuda()].cpu().numpy()
        assert np.array_equal(oracle.decode_e4m3(codes), inp.table_rows(j, rows).astype(np.float64))
    dd = inp.device_dense("cuda:0")
    dec = oracle.decode_e4m3(dd["Wk"].cpu().numpy()) * dd["k_scale"].cpu().numpy().astype(np.float64)[:, None]
    assert np.array_equal(dec, inp.Wk)


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("M", [1, 4])
def test_fp8_multibranch_matches_oracle(eb, name, M):
    wl = CASES[name]
    inp = synth.Inputs(wl, gamma="random")
    branches = [synth.branch_inputs(inp, m) for m in range(M)]
    di = DeviceInputs(inp)
    h, Wk, ks, gq, gk = _branches_dev(branches)
    ctx = eb.Engram(config_for(inp, eb))
    y = torch.full((M, wl.n_tok, wl.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    alpha = torch.empty(M, wl.n_tok, dtype=torch.float32, device="cuda")
    ctx.forward_multibranch(di.tok, di.P, di.tables, h, Wk, di.Wv, di.conv_w, y, gq=gq, gk=gk, k_scale=ks,
                            v_scale=di.v_scale, alpha_out=alpha, add_residual=True)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    ref = oracle.forward_multibranch(branches, add_residual=True)
    np.testing.assert_allclose(to_np(alpha), ref.alpha, rtol=0, atol=2e-6)
    L = wl.T - wl.t_begin
    for m in range(M):
        win = oracle.vt_windows(ref.vt[m], wl.B, L, wl.w)
        err = np.abs(to_np(y[m]) - ref.y[m])
        assert err.max() <= 2e-2, (m, err.max())
        assert not (err > bf16_bound(ref.y[m], win, inp.conv_w)).any(), m


def test_fp8_decode_with_history(eb):
    M = 2
    wl = CASES["f8a"].replace(name="f8d", B=5, T=30, t_begin=29, seed=83)
    inp = synth.Inputs(wl, gamma="random")
    branches = [synth.branch_inputs(inp, m) for m in range(M)]
    di = DeviceInputs(inp)
    h, Wk, ks, gq, gk = _branches_dev(branches)
    hist = np.stack([b.state_rows(np.arange(wl.B)) for b in branches])
    state = torch.from_numpy(hist.astype(np.float32)).cuda().contiguous()
    ctx = eb.Engram(config_for(inp, eb))
    y = torch.empty(M, wl.n_tok, wl.d, dtype=torch.bfloat16, device="cuda")
    ctx.forward_multibranch(di.tok, di.P, di.tables, h, Wk, di.Wv, di.conv_w, y, t_begin=wl.t_begin, gq=gq, gk=gk,
                            k_scale=ks, v_scale=di.v_scale, conv_state=state)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    ref = oracle.forward_multibranch(branches, hist=hist)
    for m in range(M):
        win = oracle.vt_windows(ref.vt[m], wl.B, 1, wl.w, hist[m])
        err = np.abs(to_np(y[m]) - ref.y[m])
        assert not (err > bf16_bound(ref.y[m], win, inp.conv_w)).any(), m


def test_fp8_full_size_c3_four_branches_sampled(eb):
    """c3's shapes in FP8 with four branches (5.7 GB of E4M3 tables): every
    index, and every branch's gate and Y at sampled rows."""
    import types
    M = 4
    wl = W["c3"].replace(name="c3f8", dtype="fp8")
    inp = synth.Inputs(wl, gamma="random")
    branches = [synth.branch_inputs(inp, m) for m in range(M)]
    di = DeviceInputs(inp)
    del di.h
    h, Wk, ks, gq, gk = _branches_dev(branches)
    ctx = eb.Engram(config_for(inp, eb))
    y = torch.empty(M, wl.n_tok, wl.d, dtype=torch.bfloat16, device="cuda")
    alpha = torch.empty(M, wl.n_tok, dtype=torch.float32, device="cuda")
    ctx.forward_multibranch(di.tok, di.P, di.tables, h, Wk, di.Wv, di.conv_w, y, gq=gq, gk=gk, k_scale=ks,
                            v_scale=di.v_scale, alpha_out=alpha, add_residual=True)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    canon, _ = oracle.remap(inp.tok, inp.P)
    idx_ref, _ = oracle.hash_ids(canon, wl.Vc, wl.orders, wl.K, inp.mult, inp.rows)
    idx = ctx.mb_workspace[: wl.n_tok * wl.J * 4].view(torch.int32).view(wl.n_tok, wl.J)
    assert np.array_equal(idx.cpu().numpy().view(np.uint32), idx_ref)
    pos = synth.sample_positions(wl, 48, seed=11)
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


def test_fp8_config_checks(eb):
    wl = CASES["f8a"].replace(name="f8bad", d=200)          # d not a multiple of 128
    inp = synth.Inputs(wl.replace(d=256))
    cfg = config_for(inp, eb)
    cfg.hidden = 200
    with pytest.raises(eb.EngramError) as err:
        eb.Engram(cfg)
    assert err.value.status == eb.ENGRAM_E_INVAL

"""The decode path (one new position per sequence, at most 256 sequences,
bf16) against the oracle, through engram_forward and engram_gate_conv.

These calls run the decode kernels after the retrieval: both projections in
one cluster kernel (the two halves of K on two CTA pairs, partial sums added
through distributed shared memory, the gate's row sums across clusters),
then the conv kernel, which reads and rewrites the conv state in place.
Covered: one and two 128-row accumulators (1 to 256 sequences, ragged), both
channel tile widths (64 channels: d = 256, 384, 512; 80 channels: d = 2560
on a full B200), K extents that split evenly and unevenly over the two
pairs, the indices, invalid ids (zero rows), engram_gate_conv on e, with and
without conv state and residual, bitwise determinism, and dependent against
plain launches."""

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import DeviceInputs, bf16_bound, config_for, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
BASE = W["c2"].replace(M=10007)
CASES = {
    # d_mem 512 (8 k-blocks: 2 per CTA), d 256: 64-channel tiles, 5 sequences
    "n5_d256": W["c1"].replace(name="n5_d256", B=5, T=40, t_begin=39, K=4, D=64, d=256, dtype="bf16", seed=61),
    # one accumulator, full
    "n128_d384": BASE.replace(name="n128_d384", B=128, T=9, t_begin=8, d=384, seed=62),
    # two accumulators, one row past the first
    "n129_d384": BASE.replace(name="n129_d384", B=129, T=5, t_begin=4, d=384, seed=63),
    # d 2560 (80-channel tiles on a full B200), d_mem 1024, ragged second accumulator
    "n200_d2560": BASE.replace(name="n200_d2560", B=200, T=6, t_begin=5, seed=64),
    # the c4 shape with small tables: 256 sequences, d_mem 2048 (K = 8 x 128)
    "n256_c4": W["c4"].replace(name="n256_c4", M=10007, T=64, t_begin=63, seed=65),
    # one sequence; d_mem 320 = 5 k-blocks, split 1/1/1/2 over the cluster
    "n1_uneven": W["c1"].replace(name="n1_uneven", B=1, T=3, t_begin=2, orders=(2, 3), K=5, D=32, d=512,
                                 dtype="bf16", seed=66),
}


@pytest.fixture(scope="module")
def eb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hashed_gram_embedding_02_b200 as eb
    return eb


def _decode(eb, ctx, di, state, add_residual, gamma=True):
    wl = di.wl
    y = di.empty_y()
    alpha = torch.empty(wl.n_tok, dtype=torch.float32, device=di.device)
    ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y, t_begin=wl.t_begin,
                gq=di.gq if gamma else None, gk=di.gk if gamma else None, conv_state=state, alpha_out=alpha,
                add_residual=add_residual)
    torch.cuda.synchronize()
    return y, alpha


def _kernels(eb, ctx, di, state):
    eb.engram_profile_enable(ctx.ctx, True)
    try:
        _decode(eb, ctx, di, state, True)
        return [nm for nm, _ in eb.engram_profile_read(ctx.ctx)]
    finally:
        eb.engram_profile_enable(ctx.ctx, False)


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("with_state", [True, False])
def test_decode_matches_oracle(eb, name, with_state):
    wl = CASES[name]
    assert wl.T - wl.t_begin == 1
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    add_residual = with_state
    state = inp.device_state("cuda:0").contiguous() if with_state else None
    hist = inp.state_rows(np.arange(wl.B)) if with_state else None
    y, alpha = _decode(eb, ctx, di, state, add_residual)
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    ref = oracle.forward_rows(inp, np.arange(wl.n_tok), add_residual=add_residual, hist=hist)
    # the indices of the computed position, bit-exact
    canon, _ = oracle.remap(inp.tok, inp.P)
    idx_ref, _ = oracle.hash_ids(canon, wl.Vc, wl.orders, wl.K, inp.mult, inp.rows, wl.t_begin)
    idx = ctx.workspace[: wl.n_tok * wl.J * 4].view(torch.int32).view(wl.n_tok, wl.J)
    assert np.array_equal(idx.cpu().numpy().view(np.uint32), idx_ref)
    np.testing.assert_allclose(to_np(alpha), ref.alpha, rtol=0, atol=2e-6)
    err = np.abs(to_np(y) - ref.y)
    assert err.max() <= 2e-2, err.max()
    bad = err > bf16_bound(ref.y, ref.vt_win, inp.conv_w)
    assert not bad.any(), (int(bad.sum()), float(err.max()))
    if with_state:
        # history shifted by one row, the new gated value appended
        st = state.cpu().numpy()
        np.testing.assert_array_equal(st[:, :2], hist[:, 1:].astype(np.float32))
        vt_new = ref.vt_win[:, 0]
        assert np.max(np.abs(st[:, 2] - vt_new)) <= 2.0 ** -7 * np.max(np.abs(vt_new)) + 1e-6


def test_decode_runs_the_decode_kernels(eb):
    wl = CASES["n200_d2560"]
    inp = synth.Inputs(wl)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    state = inp.device_state("cuda:0").contiguous()
    names = _kernels(eb, ctx, di, state)
    # no history transpose and no merge: the conv kernel rewrites the state in place
    assert names == ["retrieve", "gate_kv_decode", "conv_decode"], names


def test_decode_invalid_ids_read_zero_rows(eb):
    """Ids outside the vocabulary in the n-gram windows of some sequences:
    every order whose window holds one reads zero rows and the status word
    says ENGRAM_ERR_TOKEN."""
    wl = CASES["n200_d2560"]
    inp = synth.Inputs(wl, gamma="random")
    t = wl.t_begin
    inp.tok[3, t] = wl.V + 5        # every order of sequence 3
    inp.tok[7, t - 1] = -3          # both orders of sequence 7
    inp.tok[9, t - 2] = wl.V        # order 3 only (tables 8-15, the second half of K)
    inp.tok[150, t - 2] = -1        # the same in the second 128-row block
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    state = inp.device_state("cuda:0").contiguous()
    hist = inp.state_rows(np.arange(wl.B))
    y, alpha = _decode(eb, ctx, di, state, True)
    st, flags = ctx.status()
    assert flags == eb.ENGRAM_ERR_TOKEN, (st, flags)
    ref = oracle.forward_rows(inp, np.arange(wl.n_tok), add_residual=True, hist=hist)
    np.testing.assert_allclose(to_np(alpha), ref.alpha, rtol=0, atol=2e-6)
    err = np.abs(to_np(y) - ref.y)
    bad = err > bf16_bound(ref.y, ref.vt_win, inp.conv_w)
    assert not bad.any(), (int(bad.sum()), float(err.max()))
    idx = ctx.workspace[: wl.n_tok * wl.J * 4].view(torch.int32).view(wl.n_tok, wl.J).cpu().numpy().view(np.uint32)
    assert (idx[3] == eb.ENGRAM_INVALID_INDEX).all() and (idx[7] == eb.ENGRAM_INVALID_INDEX).all()
    assert (idx[9, : wl.K] != eb.ENGRAM_INVALID_INDEX).all() and (idx[9, wl.K:] == eb.ENGRAM_INVALID_INDEX).all()


@pytest.mark.parametrize("name", ["n200_d2560", "n5_d256"])
def test_gate_conv_decode_from_e(eb, name):
    """engram_gate_conv on one position per sequence runs the same decode
    kernels on the caller's e (here made on the device by engram_hash and
    engram_gather)."""
    wl = CASES[name]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    n = wl.n_tok
    idx = torch.empty(n, wl.J, dtype=torch.int32, device="cuda")
    eb.engram_hash(ctx.ctx, di.tok, di.P, wl.B, wl.T, wl.T, wl.t_begin, idx)
    e = torch.empty(n, wl.J * wl.D, dtype=torch.bfloat16, device="cuda")
    eb.engram_gather(ctx.ctx, idx, n, di.tables, e)
    ws_bytes = eb.engram_workspace_bytes(ctx.ctx, wl.B, 1)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    state = inp.device_state("cuda:0").contiguous()
    hist = inp.state_rows(np.arange(wl.B))
    y = di.empty_y()
    alpha = torch.empty(n, dtype=torch.float32, device="cuda")
    eb.engram_profile_enable(ctx.ctx, True)
    try:
        eb.engram_gate_conv(ctx.ctx, e, di.h, di.Wk, di.Wv, di.gq, di.gk, di.conv_w, wl.B, 1, state, y, alpha, 1,
                            ws, ws_bytes)
        torch.cuda.synchronize()
        names = [nm for nm, _ in eb.engram_profile_read(ctx.ctx)]
    finally:
        eb.engram_profile_enable(ctx.ctx, False)
    assert names == ["gate_kv_decode", "conv_decode"], names
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    ref = oracle.forward_rows(inp, np.arange(n), add_residual=True, hist=hist)
    np.testing.assert_allclose(to_np(alpha), ref.alpha, rtol=0, atol=2e-6)
    err = np.abs(to_np(y) - ref.y)
    bad = err > bf16_bound(ref.y, ref.vt_win, inp.conv_w)
    assert not bad.any(), (int(bad.sum()), float(err.max()))


def test_decode_without_gains(eb):
    wl = CASES["n129_d384"]
    inp = synth.Inputs(wl)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    y, alpha = _decode(eb, ctx, di, None, False, gamma=False)
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    inp.gq = np.ones_like(inp.gq)
    inp.gk = np.ones_like(inp.gk)
    ref = oracle.forward_rows(inp, np.arange(wl.n_tok))
    np.testing.assert_allclose(to_np(alpha), ref.alpha, rtol=0, atol=2e-6)
    assert np.abs(to_np(y) - ref.y).max() <= 2e-2


@pytest.mark.parametrize("name", ["n256_c4", "n5_d256"])
def test_decode_deterministic_and_dependent_launches_match_plain(eb, name):
    """Same bits from two dependent-launch runs and from a run with kernel
    timing on (plain launches with events between them).  A decode on other
    hidden states runs first, so a conv kernel that read v or alpha before the
    projection kernel completed would see different values."""
    wl = CASES[name]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    s0 = inp.device_state("cuda:0").contiguous()
    y0 = di.empty_y()
    ctx.forward(di.tok, di.P, di.tables, (di.h * 3).contiguous(), di.Wk, di.Wv, di.conv_w, y0, t_begin=wl.t_begin,
                gq=di.gq, gk=di.gk, conv_state=s0.clone(), add_residual=True)
    outs = []
    for prof in (False, False, True):
        st = s0.clone()
        eb.engram_profile_enable(ctx.ctx, prof)
        try:
            y, a = _decode(eb, ctx, di, st, True)
        finally:
            eb.engram_profile_enable(ctx.ctx, False)
        outs.append((y, a, st))
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    for y, a, st in outs[1:]:
        assert torch.equal(y, outs[0][0]) and torch.equal(a, outs[0][1]) and torch.equal(st, outs[0][2])


def test_two_decode_steps_match_a_prefill(eb):
    """Prefill T-2 positions, then decode t = T-2 and t = T-1 one at a time
    through the conv state: each decode row equals the prefill row over all
    T positions (same v and alpha arithmetic up to a bf16 flip of v)."""
    wl = CASES["n5_d256"].replace(t_begin=0)
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    L = wl.T
    y_full = di.empty_y()
    ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y_full, gq=di.gq, gk=di.gk)
    state = torch.zeros(wl.B, wl.w - 1, wl.d, dtype=torch.float32, device="cuda")
    h_rows = di.h.view(wl.B, L, wl.d)
    y1 = torch.empty(wl.B * (L - 2), wl.d, dtype=di.dtype, device="cuda")
    ctx.forward(di.tok[:, : L - 2], di.P, di.tables, h_rows[:, : L - 2].contiguous().view(-1, wl.d), di.Wk, di.Wv,
                di.conv_w, y1, gq=di.gq, gk=di.gk, conv_state=state)
    full = y_full.view(wl.B, L, wl.d)
    for t in (L - 2, L - 1):
        y2 = torch.empty(wl.B, wl.d, dtype=di.dtype, device="cuda")
        ctx.forward(di.tok[:, : t + 1], di.P, di.tables, h_rows[:, t].contiguous(), di.Wk, di.Wv, di.conv_w, y2,
                    t_begin=t, gq=di.gq, gk=di.gk, conv_state=state)
        torch.cuda.synchronize()
        assert ctx.status() == (eb.ENGRAM_OK, 0)
        diff = (y2.float() - full[:, t].float()).abs().max().item()
        assert diff <= 2e-2, (t, diff)

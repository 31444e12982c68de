"""engram_forward_noalloc: the forward for callers that cannot allocate device
memory (an engine callback where allocation is forbidden, a process whose
device memory belongs to another allocator, a loop that cannot take
cudaMalloc's implicit synchronisation).  It runs out of the library's static
device scratch array; its results must match engram_forward with a caller
workspace, call after call, since the array keeps the previous call's
contents.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test; it also passes on its own in a
fresh process (the first call on the device does the scratch set-up)."""

import numpy as np
import pytest

import synth
from gpu_helpers import DeviceInputs, config_for, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
CASES = {
    # bf16, fused tensor-core path (two tcgen05 passes), ragged rows
    "b3": W["c2"].replace(name="b3", B=2, T=333, M=10007, d=512, seed=14),
    # fp32, CUDA-core path
    "c1": W["c1"],
}


@pytest.fixture(scope="module")
def eb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hashed_gram_embedding_02_b200 as eb
    return eb


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_workspace_forward_twice(eb, name):
    wl = CASES[name]
    inp = synth.Inputs(wl, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    y_ref = di.empty_y()
    a_ref = torch.empty(wl.n_tok, dtype=torch.float32, device="cuda")
    ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y_ref, gq=di.gq, gk=di.gk,
                alpha_out=a_ref, add_residual=True)
    # same kernels, inputs and launches as the workspace forward, which is
    # deterministic: any difference would be scratch aliasing, so equality
    for call in range(2):
        y = torch.full_like(y_ref, float("nan"))
        a = torch.full_like(a_ref, float("nan"))
        eb.engram_forward_noalloc(ctx.ctx, di.tok, wl.B, wl.T, wl.T, 0, di.P, di.tables, di.h, di.Wk, di.Wv, di.gq,
                                  di.gk, di.conv_w, None, y, a, 1)
        torch.cuda.synchronize()
        assert ctx.status() == (eb.ENGRAM_OK, 0)
        assert torch.equal(y, y_ref), (call, float(np.max(np.abs(to_np(y) - to_np(y_ref)))))
        assert torch.equal(a, a_ref), call


def test_noalloc_with_conv_history_twice(eb):
    """Decode-style call (one new position per sequence, history in conv_state)."""
    wl = W["c1"].replace(name="dec", B=3, T=40, t_begin=39, K=4, D=64, d=256, dtype="bf16", seed=31)
    inp = synth.Inputs(wl)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    state0 = inp.device_state("cuda:0").contiguous()
    s_ref = state0.clone()
    y_ref = di.empty_y()
    ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y_ref, t_begin=wl.t_begin, conv_state=s_ref)
    for call in range(2):
        s = state0.clone()
        y = torch.full_like(y_ref, float("nan"))
        eb.engram_forward_noalloc(ctx.ctx, di.tok, wl.B, wl.T, wl.T, wl.t_begin, di.P, di.tables, di.h, di.Wk,
                                  di.Wv, None, None, di.conv_w, s, y, None, 0)
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref), call
        assert torch.equal(s, s_ref), call


def test_noalloc_rejects_batches_beyond_the_static_scratch(eb):
    from hashed_gram_embedding_02_b200 import binding
    wl = W["c2"].replace(M=10007)
    inp = synth.Inputs(wl.replace(B=1, T=8))
    ctx = eb.Engram(config_for(inp, eb))
    big_T = 65536                       # needs far more than the static scratch
    assert eb.engram_workspace_bytes(ctx.ctx, 4, big_T) > eb.ENGRAM_NOALLOC_SCRATCH_BYTES
    tok = torch.zeros(4, big_T, dtype=torch.int32, device="cuda")
    y = torch.zeros(1, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.EngramError) as ei:
        eb.engram_forward_noalloc(ctx.ctx, tok, 4, big_T, big_T, 0, tok, y, y, y, y, None, None,
                                  torch.zeros(4, device="cuda"), None, y, None, 0)
    assert ei.value.status == binding.ENGRAM_E_NOMEM
    assert "static scratch" in str(ei.value)

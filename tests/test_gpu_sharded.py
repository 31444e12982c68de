"""Tables split into shards: the forward that reads every row from the
shard owning it equals the forward on the whole table array, bit for bit
(indices, e and Y; the kernels after the retrieval are the same).

On one GPU the shards are separate device allocations (several shards per
GPU); a second process on the same GPU exports its shards through CUDA IPC
and this process maps them, which is the path a job with one process per GPU
takes (there each peer's shard is another GPU's memory, read over NVLink).
Nothing here waits on another process's kernels."""

import multiprocessing as mp

import numpy as np
import pytest

import synth
from gpu_helpers import DeviceInputs, config_for

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
CASE = W["c2"].replace(name="sh", B=2, T=333, M=10007, d=512, seed=51)


@pytest.fixture(scope="module")
def eb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hashed_gram_embedding_02_b200 as eb
    return eb


def _shards(eb, ctx, tables, n_shards):
    """The shards as separate allocations, filled from the whole table array."""
    flat = tables.reshape(-1, tables.shape[-1])
    out = []
    for g in range(n_shards):
        lo, cnt = eb.engram_shard_range(ctx.ctx, n_shards, g)
        out.append(flat[lo:lo + cnt].clone() if cnt else None)
    return out


def _ws_e(ctx, wl):
    """idx and e of the last forward, from the context's workspace (idx | e)."""
    idx_bytes = wl.n_tok * wl.J * 4
    idx = ctx.workspace[:idx_bytes].view(torch.int32).view(wl.n_tok, wl.J).clone()
    e_off = (idx_bytes + 255) // 256 * 256
    e = ctx.workspace[e_off:e_off + wl.n_tok * wl.d_mem * 2].view(torch.bfloat16).view(wl.n_tok, wl.d_mem).clone()
    return idx, e


def test_shard_ranges_cover_the_rows(eb):
    inp = synth.Inputs(CASE)
    ctx = eb.Engram(config_for(inp, eb))
    R = CASE.J * CASE.M
    for n in (1, 2, 3, 7, 16):
        ranges = [eb.engram_shard_range(ctx.ctx, n, g) for g in range(n)]
        pos = 0
        for lo, cnt in ranges:
            assert lo == pos and cnt >= 0
            pos += cnt
        assert pos == R
        assert max(c for _, c in ranges) == -(-R // n)
    with pytest.raises(eb.EngramError):
        eb.engram_shard_range(ctx.ctx, 17, 0)


@pytest.mark.parametrize("n_shards", [1, 2, 3, 5, 8, 16])
def test_sharded_forward_equals_forward(eb, n_shards):
    inp = synth.Inputs(CASE, gamma="random")
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    y_ref = di.empty_y()
    a_ref = torch.empty(CASE.n_tok, dtype=torch.float32, device="cuda")
    ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y_ref, gq=di.gq, gk=di.gk, alpha_out=a_ref,
                add_residual=True)
    torch.cuda.synchronize()
    idx_ref, e_ref = _ws_e(ctx, CASE)
    shards = _shards(eb, ctx, di.tables, n_shards)
    ptrs = [s.data_ptr() if s is not None else 0 for s in shards]
    y = torch.full_like(y_ref, float("nan"))
    a = torch.full_like(a_ref, float("nan"))
    ctx.forward_sharded(di.tok, di.P, ptrs, di.h, di.Wk, di.Wv, di.conv_w, y, gq=di.gq, gk=di.gk, alpha_out=a,
                        add_residual=True)
    torch.cuda.synchronize()
    assert ctx.status() == (eb.ENGRAM_OK, 0)
    idx, e = _ws_e(ctx, CASE)
    assert torch.equal(idx, idx_ref)
    assert torch.equal(e, e_ref)
    assert torch.equal(y, y_ref) and torch.equal(a, a_ref)


def test_sharded_decode_with_state(eb):
    wl = CASE.replace(name="shd", B=5, T=64, t_begin=63)
    inp = synth.Inputs(wl)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    s0 = inp.device_state("cuda:0").contiguous()
    s_ref, s = s0.clone(), s0.clone()
    y_ref, y = di.empty_y(), di.empty_y()
    ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y_ref, t_begin=wl.t_begin, conv_state=s_ref)
    shards = _shards(eb, ctx, di.tables, 4)
    ctx.forward_sharded(di.tok, di.P, [x.data_ptr() for x in shards], di.h, di.Wk, di.Wv, di.conv_w, y,
                        t_begin=wl.t_begin, conv_state=s)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref) and torch.equal(s, s_ref)


def test_sharded_rejects_bad_lists(eb):
    inp = synth.Inputs(CASE)
    di = DeviceInputs(inp)
    ctx = eb.Engram(config_for(inp, eb))
    y = di.empty_y()
    shards = _shards(eb, ctx, di.tables, 2)
    with pytest.raises(eb.EngramError) as err:
        ctx.forward_sharded(di.tok, di.P, [shards[0].data_ptr(), 0], di.h, di.Wk, di.Wv, di.conv_w, y)
    assert err.value.status == eb.ENGRAM_E_INVAL
    with pytest.raises(eb.EngramError):
        ctx.forward_sharded(di.tok, di.P, [shards[0].data_ptr() + 2, shards[1].data_ptr()], di.h, di.Wk, di.Wv,
                            di.conv_w, y)
    with pytest.raises(eb.EngramError):
        ctx.forward_sharded(di.tok, di.P, [shards[0].data_ptr()] * 17, di.h, di.Wk, di.Wv, di.conv_w, y)


# ---------------------------------------------------------------- two processes, CUDA IPC

def _owner(conn, n_shards, owned):
    """Child process: builds the tables, keeps the shards in `owned`, exports
    them, and holds them until the parent says it is done."""
    import torch
    import hashed_gram_embedding_02_b200 as eb
    from gpu_helpers import config_for as cfg_for
    torch.cuda.set_device(0)
    inp = synth.Inputs(CASE)
    ctx = eb.Engram(cfg_for(inp, eb))
    flat = inp.device_tables("cuda:0").reshape(-1, CASE.D)
    keep, out = [], {}
    for g in owned:
        lo, cnt = eb.engram_shard_range(ctx.ctx, n_shards, g)
        t = torch.empty(cnt + 3, CASE.D, dtype=torch.bfloat16, device="cuda")   # the shard at an offset
        t[3:] = flat[lo:lo + cnt]
        keep.append(t)
        out[g] = eb.engram_ipc_export(t[3:].data_ptr())
    torch.cuda.synchronize()
    conn.send(out)
    conn.recv()            # the parent has closed its mappings
    conn.close()


def test_shards_of_another_process_through_ipc(eb):
    n_shards, owned = 4, (1, 3)
    ctx_mp = mp.get_context("spawn")
    parent, child = ctx_mp.Pipe()
    p = ctx_mp.Process(target=_owner, args=(child, n_shards, owned))
    p.start()
    try:
        exported = parent.recv()
        inp = synth.Inputs(CASE, gamma="random")
        di = DeviceInputs(inp)
        ctx = eb.Engram(config_for(inp, eb))
        y_ref = di.empty_y()
        ctx.forward(di.tok, di.P, di.tables, di.h, di.Wk, di.Wv, di.conv_w, y_ref, gq=di.gq, gk=di.gk,
                    add_residual=True)
        local = _shards(eb, ctx, di.tables, n_shards)
        ptrs, bases = [], []
        for g in range(n_shards):
            if g in exported:
                handle, off = exported[g]
                assert off % 16 == 0
                ptr, base = eb.engram_ipc_open(handle, off)
                ptrs.append(ptr)
                bases.append(base)
            else:
                ptrs.append(local[g].data_ptr())
        y = torch.full_like(y_ref, float("nan"))
        ctx.forward_sharded(di.tok, di.P, ptrs, di.h, di.Wk, di.Wv, di.conv_w, y, gq=di.gq, gk=di.gk,
                            add_residual=True)
        torch.cuda.synchronize()
        assert ctx.status() == (eb.ENGRAM_OK, 0)
        assert torch.equal(y, y_ref)
        for b in bases:
            eb.engram_ipc_close(b)
    finally:
        parent.send("done")
        p.join(timeout=120)
        if p.is_alive():
            p.kill()
    assert p.exitcode == 0

"""Engram conditional-memory forward path for NVIDIA B200 (sm_100a).

The compute lives in ``libengram.so`` (CUDA kernels behind the C ABI declared
in ``include/engram.h``); :mod:`.binding` is its ctypes binding with the same
function names, and :class:`Engram` is a small convenience owner of a context
plus its workspace.  PyTorch is used only for device memory and streams.
"""

from __future__ import annotations

from typing import Optional

from .binding import (  # noqa: F401  (re-exported C ABI names)
    ENGRAM_BF16, ENGRAM_F32, ENGRAM_FP8, ENGRAM_ERR_CANON, ENGRAM_ERR_INDEX, ENGRAM_ERR_TIMEOUT, ENGRAM_ERR_TOKEN,
    ENGRAM_E_CUDA, ENGRAM_E_DEVICE, ENGRAM_E_HOST, ENGRAM_E_INVAL, ENGRAM_E_NOMEM, ENGRAM_E_TIMEOUT,
    ENGRAM_E_UNSUPPORTED,
    ENGRAM_INVALID_INDEX, ENGRAM_OK, EXPORTS, LIB_PATH, EngramError, engram_config, engram_conv, engram_create,
    ENGRAM_NOALLOC_SCRATCH_BYTES, engram_destroy, engram_device_status, engram_forward, engram_forward_noalloc,
    engram_forward_host, engram_gate_conv, engram_gather, engram_gather_staged, engram_hash, engram_host_dedupe,
    engram_host_fetch, engram_host_tier_create, engram_host_tier_destroy, engram_host_tier_stats,
    engram_host_workspace_bytes, engram_pack_rows, engram_debug_stall_next, engram_host_tier_debug,
    ENGRAM_INJECT_LIST_WAIT, ENGRAM_INJECT_PACK_ABANDON, engram_host_cache_enable, engram_host_cache_reset,
    engram_host_cache_stats, engram_shard_range, engram_forward_sharded, engram_ipc_export, engram_ipc_open,
    engram_ipc_close, ENGRAM_IPC_HANDLE_BYTES, ENGRAM_MAX_SHARDS, engram_multibranch_workspace_bytes,
    engram_forward_multibranch, ENGRAM_MAX_BRANCHES, engram_table_grad_workspace_bytes, engram_table_grad,
    engram_table_sgd, engram_host_tier_map, engram_grad_route_workspace_bytes, engram_grad_route,
    engram_grad_combine_workspace_bytes, engram_grad_combine, engram_shard_sgd,
    engram_last_error, engram_profile_enable, engram_profile_read, engram_project, engram_remap, engram_strerror,
    engram_workspace_bytes, make_config)


class Engram:
    """Owns one engram_ctx (bound to the current device) and a workspace,
    grown on demand (or reserved up front for B sequences of L rows)."""

    def __init__(self, cfg: engram_config, B: int = 0, L: int = 0):
        import torch
        self.cfg = cfg
        self.ctx = engram_create(cfg)
        self.device = torch.device("cuda", torch.cuda.current_device())
        self.workspace = None
        self.workspace_bytes = 0
        if B and L:
            self.reserve(B, L)

    def reserve(self, B: int, L: int):
        import torch
        need = engram_workspace_bytes(self.ctx, B, L)
        if need > self.workspace_bytes:
            self.workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
            self.workspace_bytes = need

    def close(self):
        if self.ctx:
            engram_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def G(self) -> int:
        return (self.cfg.hidden + 127) // 128

    def forward(self, tok, P, tables, h, Wk, Wv, conv_w, y, *, t_begin: int = 0, gq=None, gk=None,
                conv_state=None, alpha_out=None, add_residual: bool = False, stream=None):
        B, T = tok.shape[0], tok.shape[1]
        self.reserve(B, T - t_begin)
        engram_forward(self.ctx, tok, B, T, tok.stride(0), t_begin, P, tables, h, Wk, Wv, gq, gk, conv_w,
                       conv_state, y, alpha_out, add_residual, self.workspace, self.workspace_bytes, stream)
        return y

    def forward_multibranch(self, tok, P, tables, h, Wk, Wv, conv_w, y, *, t_begin: int = 0, gq=None, gk=None,
                            k_scale=None, v_scale=None, conv_state=None, alpha_out=None, add_residual: bool = False,
                            stream=None):
        """M-branch forward: h [M][n][d], Wk [M][d][d_mem], gq/gk [M][d],
        conv_state [M][B][w-1][d], y [M][n][d], alpha_out [M][n]."""
        import torch
        M = h.shape[0]
        B, T = tok.shape[0], tok.shape[1]
        need = engram_multibranch_workspace_bytes(self.ctx, M, B, T - t_begin)
        if need > getattr(self, "mb_workspace_bytes", 0):
            self.mb_workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
            self.mb_workspace_bytes = need
        engram_forward_multibranch(self.ctx, M, tok, B, T, tok.stride(0), t_begin, P, tables, h, Wk, Wv, gq, gk,
                                   k_scale, v_scale, conv_w, conv_state, y, alpha_out, add_residual, self.mb_workspace,
                                   self.mb_workspace_bytes, stream)
        return y

    def forward_sharded(self, tok, P, shard_ptrs, h, Wk, Wv, conv_w, y, *, t_begin: int = 0, gq=None, gk=None,
                        conv_state=None, alpha_out=None, add_residual: bool = False, stream=None):
        """The forward with the tables split into shards (device pointers
        valid on this GPU, in shard order: ShardedTables.ptrs)."""
        B, T = tok.shape[0], tok.shape[1]
        self.reserve(B, T - t_begin)
        engram_forward_sharded(self.ctx, tok, B, T, tok.stride(0), t_begin, P, shard_ptrs, h, Wk, Wv, gq, gk, conv_w,
                               conv_state, y, alpha_out, add_residual, self.workspace, self.workspace_bytes, stream)
        return y

    def forward_host(self, tok_host, P, tables, h_host, Wk, Wv, conv_w, y_host, *, t_begin: int = 0, gq=None,
                     gk=None, conv_state=None, add_residual: bool = False, chunk_rows: int = 0, stream=None):
        """The forward with tok, h and y in host memory (pinned CPU tensors
        overlap their copies with the compute); returns y_host, complete once
        the stream is synchronised."""
        import torch
        B, T = tok_host.shape[0], tok_host.shape[1]
        need = engram_host_workspace_bytes(self.ctx, B, T, t_begin, chunk_rows)
        if need > getattr(self, "host_workspace_bytes", 0):
            self.host_workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
            self.host_workspace_bytes = need
        engram_forward_host(self.ctx, tok_host, B, T, tok_host.stride(0), t_begin, P, tables, h_host, Wk, Wv, gq, gk,
                            conv_w, conv_state, y_host, add_residual, chunk_rows, self.host_workspace,
                            self.host_workspace_bytes, stream)
        return y_host

    def table_grad(self, idx, d_e, stream=None):
        """Sparse gradient of the tables from dL/de: (rows [U] int64 global
        rows, grad [U][D] fp32), U read back from the device (a sync)."""
        import torch
        n_tok = idx.shape[0]
        n = max(1, n_tok * idx.shape[1])
        need = engram_table_grad_workspace_bytes(self.ctx, n_tok)
        ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        rows = torch.empty(n, dtype=torch.int64, device=self.device)
        grad = torch.empty(n, self.cfg.row_dim, dtype=torch.float32, device=self.device)
        cnt = torch.zeros(1, dtype=torch.int64, device=self.device)
        engram_table_grad(self.ctx, idx, n_tok, d_e, rows, grad, cnt, ws, need, stream)
        U = int(cnt.item())
        return rows[:U], grad[:U], cnt

    def grad_route(self, rows, grad, n_pairs, n_shards: int, stream=None):
        """This rank's (row, gradient) pairs split by the shard that owns the
        row: (send_rows, send_grad, send_counts), the counts an int64 [n_shards]
        tensor on the device, the segments in shard order."""
        import torch
        max_rows = rows.shape[0]
        send_rows = torch.empty(max(1, max_rows), dtype=torch.int64, device=self.device)
        send_grad = torch.empty(max(1, max_rows), self.cfg.row_dim, dtype=torch.float32, device=self.device)
        send_counts = torch.empty(n_shards, dtype=torch.int64, device=self.device)
        need = engram_grad_route_workspace_bytes(self.ctx)
        ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        engram_grad_route(self.ctx, n_shards, rows, grad, n_pairs, max_rows, send_rows, send_grad, send_counts, ws,
                          need, stream)
        return send_rows, send_grad, send_counts

    def grad_combine(self, pair_rows, pair_grad, n_shards: int, shard: int, stream=None):
        """The pairs received by shard `shard`, summed per row: (rows [U]
        int64 global rows, grad [U][D] fp32, count), U read back (a sync)."""
        import torch
        n = pair_rows.shape[0]
        need = engram_grad_combine_workspace_bytes(self.ctx, n)
        ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        rows = torch.empty(max(1, n), dtype=torch.int64, device=self.device)
        grad = torch.empty(max(1, n), self.cfg.row_dim, dtype=torch.float32, device=self.device)
        cnt = torch.zeros(1, dtype=torch.int64, device=self.device)
        engram_grad_combine(self.ctx, n_shards, shard, pair_rows, pair_grad, n, rows, grad, cnt, ws, need, stream)
        U = int(cnt.item())
        return rows[:U], grad[:U], cnt

    def shard_sgd(self, n_shards: int, shard: int, rows, grad, n_unique, shard_table, lr: float, stream=None):
        """shard_table[row - first] -= lr * grad for the listed global rows."""
        engram_shard_sgd(self.ctx, n_shards, shard, rows, grad, n_unique, rows.shape[0], shard_table, lr, stream)

    def status(self, stream=None):
        return engram_device_status(self.ctx, stream)


class HostTier:
    """Owns one engram_host_tier: tables in host memory, rows fetched per
    batch (engram_host_dedupe -> engram_host_fetch -> engram_gather_staged)."""

    def __init__(self, engram: "Engram", host_tables, max_lookups: int, n_threads: int = 8):
        self.engram = engram
        self.host_tables = host_tables          # keeps the host memory alive
        self.tier = engram_host_tier_create(engram.ctx, host_tables, max_lookups, n_threads)

    def close(self):
        if self.tier:
            engram_host_tier_destroy(self.tier)
            self.tier = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def dedupe(self, idx, n_tok: int, stream=None):
        engram_host_dedupe(self.tier, idx, n_tok, stream)

    def fetch(self, side_stream) -> int:
        return engram_host_fetch(self.tier, side_stream)

    def gather(self, n_tok: int, e_cat, stream=None):
        engram_gather_staged(self.tier, n_tok, e_cat, stream)
        return e_cat

    def stats(self):
        return engram_host_tier_stats(self.tier)

    def map_tables(self):
        """Fetch rows with a GPU kernel reading the mapped host tables."""
        engram_host_tier_map(self.tier)

    def enable_cache(self, capacity_rows: int, min_count: int = 2):
        engram_host_cache_enable(self.tier, capacity_rows, min_count)

    def reset_cache(self, stream=None):
        engram_host_cache_reset(self.tier, stream)

    def cache_stats(self):
        return engram_host_cache_stats(self.tier)

    def debug(self, inject: int, wait_limit_s: float):
        engram_host_tier_debug(self.tier, inject, wait_limit_s)


def exchange_shards(local_ptr: int, rank: int, world: int, all_gather, export=None, open_=None):
    """Shard pointers valid on this rank's GPU for every rank's shard.

    One process per GPU; rank r holds shard r at the device pointer
    ``local_ptr``.  Each rank exports its shard (an IPC handle and offset),
    ``all_gather(obj) -> [obj of rank 0, ..., obj of rank world-1]`` collects
    every rank's export (``torch.distributed.all_gather_object`` in a job),
    and each rank maps the others' shards into its own address space.
    Returns (pointers in shard order, mapping bases to close later).  The
    export/open functions default to the library's IPC calls; the host logic
    is the same with any pair."""
    export = engram_ipc_export if export is None else export
    open_ = engram_ipc_open if open_ is None else open_
    mine = export(local_ptr) if world > 1 else None
    every = all_gather(mine) if world > 1 else [mine]
    if len(every) != world:
        raise RuntimeError(f"expected {world} shard exports, got {len(every)}")
    ptrs, bases = [], []
    for g in range(world):
        if g == rank:
            ptrs.append(int(local_ptr))
            continue
        handle, offset = every[g]
        ptr, base = open_(handle, offset)
        ptrs.append(ptr)
        bases.append(base)
    return ptrs, bases


class ShardedTables:
    """This rank's shard of the tables (rank r of ``world`` holds shard r, the
    global rows ``engram_shard_range`` gives it) and the pointers of every
    shard on this rank's GPU.  ``fill(first_row, n_rows, out)`` writes the
    shard's rows into ``out`` ([n_rows][D] on the device).  Mappings of
    other ranks' shards are closed by :meth:`close`; all ranks must keep
    their shard alive until every rank is done with it (a barrier)."""

    def __init__(self, engram: "Engram", world: int, rank: int, row_dim: int, dtype, device, fill, all_gather=None,
                 export=None, open_=None, close=None):
        import torch
        self.first, self.rows = engram_shard_range(engram.ctx, world, rank)
        self.local = torch.empty(max(1, self.rows), row_dim, dtype=dtype, device=device)
        if self.rows:
            fill(self.first, self.rows, self.local[: self.rows])
        torch.cuda.synchronize(device)
        self._close = engram_ipc_close if close is None else close
        self.ptrs, self._bases = exchange_shards(self.local.data_ptr(), rank, world, all_gather, export, open_)

    def close(self):
        for b in self._bases:
            self._close(b)
        self._bases = []


def all_to_all_pairs(send_rows, send_grad, send_counts, all_to_all_single=None):
    """The backward's exchange of (row, gradient) pairs between the ranks.

    ``send_counts[g]`` pairs of this rank are for rank g (one shard per rank),
    in segments of ``send_rows`` / ``send_grad`` in rank order (what
    :meth:`Engram.grad_route` writes).  First the counts go round (one int64
    from every rank to every rank), then the segments, with the split sizes
    those counts give.  Returns (recv_rows, recv_grad, recv_counts as a host
    list): the pairs sent to this rank by rank 0, then rank 1, and so on.
    ``all_to_all_single`` defaults to ``torch.distributed``'s (NCCL between
    GPUs, gloo on CPU); reading the counts on the host is a sync."""
    import torch
    if all_to_all_single is None:
        import torch.distributed as dist
        all_to_all_single = dist.all_to_all_single
    recv_counts = torch.empty_like(send_counts)
    all_to_all_single(recv_counts, send_counts)
    in_split = [int(x) for x in send_counts.tolist()]
    out_split = [int(x) for x in recv_counts.tolist()]
    if min(in_split + out_split, default=0) < 0:
        raise RuntimeError(f"negative pair count in {in_split} / {out_split}")
    n_send, n_recv = sum(in_split), sum(out_split)
    if n_send > send_rows.shape[0]:
        raise RuntimeError(f"{n_send} pairs to send, the send buffers hold {send_rows.shape[0]}")
    D = send_grad.shape[1]
    recv_rows = torch.empty(n_recv, dtype=send_rows.dtype, device=send_rows.device)
    recv_grad = torch.empty(n_recv, D, dtype=send_grad.dtype, device=send_grad.device)
    all_to_all_single(recv_rows, send_rows[:n_send], out_split, in_split)
    all_to_all_single(recv_grad, send_grad[:n_send], out_split, in_split)
    return recv_rows, recv_grad, out_split


def sharded_table_step(engram: Engram, tables: ShardedTables, idx, d_e, lr: float, rank: int, world: int,
                       all_to_all_single=None):
    """One update of sharded tables from this rank's batch: the sparse
    gradient of the rows the batch looked up (engram_table_grad), routed to
    the ranks that own them (engram_grad_route), exchanged
    (:func:`all_to_all_pairs`), summed per row in rank order
    (engram_grad_combine) and applied to this rank's shard
    (engram_shard_sgd).  Every rank calls it with its own batch; returns the
    (rows, gradient) applied to this rank's shard."""
    rows, grad, cnt = engram.table_grad(idx, d_e)
    send_rows, send_grad, send_counts = engram.grad_route(rows, grad, cnt, world)
    recv_rows, recv_grad, _ = all_to_all_pairs(send_rows, send_grad, send_counts, all_to_all_single)
    r, g, u = engram.grad_combine(recv_rows, recv_grad, world, rank)
    engram.shard_sgd(world, rank, r, g, u, tables.local, lr)
    return r, g

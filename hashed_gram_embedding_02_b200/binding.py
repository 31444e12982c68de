"""ctypes binding of libengram.so: same names as the C ABI, argument
marshalling only.

Tensors are torch tensors on the context's device (PyTorch provides device
memory and streams); every step of the path runs in the library's kernels.
Each wrapper raises :class:`EngramError` when the C call returns a non-zero
status.  Importing this module without the built library raises at once:
there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libengram.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m hashed_gram_embedding_02_b200.build` "
                      "or __graft_entry__.build(); the Engram path has no CPU fallback")

_lib = ctypes.CDLL(LIB_PATH)

ENGRAM_OK, ENGRAM_E_INVAL, ENGRAM_E_CUDA, ENGRAM_E_NOMEM, ENGRAM_E_UNSUPPORTED, ENGRAM_E_TIMEOUT, \
    ENGRAM_E_HOST, ENGRAM_E_DEVICE = range(8)
ENGRAM_F32, ENGRAM_BF16, ENGRAM_FP8 = 0, 1, 2
ENGRAM_ERR_TOKEN, ENGRAM_ERR_CANON, ENGRAM_ERR_INDEX, ENGRAM_ERR_TIMEOUT = 0x1, 0x2, 0x4, 0x8
ENGRAM_INJECT_LIST_WAIT, ENGRAM_INJECT_PACK_ABANDON = 0x1, 0x2
ENGRAM_INVALID_INDEX = 0xFFFFFFFF
ENGRAM_MAX_TABLES = 32
ENGRAM_PART_GROUP = 128

# exported symbol names declared in include/engram.h
EXPORTS = ("engram_create", "engram_destroy", "engram_strerror", "engram_last_error", "engram_workspace_bytes",
           "engram_profile_enable", "engram_profile_read", "engram_device_status", "engram_remap", "engram_hash",
           "engram_gather", "engram_project", "engram_conv", "engram_gate_conv", "engram_forward",
           "engram_forward_noalloc", "engram_host_workspace_bytes", "engram_forward_host", "engram_host_tier_create",
           "engram_host_tier_destroy", "engram_host_dedupe", "engram_host_fetch", "engram_gather_staged",
           "engram_host_tier_stats", "engram_pack_rows", "engram_debug_stall_next", "engram_host_tier_debug",
           "engram_host_cache_enable", "engram_host_cache_reset", "engram_host_cache_stats",
           "engram_shard_range", "engram_forward_sharded", "engram_ipc_export", "engram_ipc_open", "engram_ipc_close",
           "engram_multibranch_workspace_bytes", "engram_forward_multibranch", "engram_table_grad_workspace_bytes",
           "engram_table_grad", "engram_table_sgd", "engram_host_tier_map", "engram_grad_route_workspace_bytes",
           "engram_grad_route", "engram_grad_combine_workspace_bytes", "engram_grad_combine", "engram_shard_sgd")
ENGRAM_MAX_BRANCHES = 4
ENGRAM_IPC_HANDLE_BYTES = 64
ENGRAM_MAX_SHARDS = 16
ENGRAM_NOALLOC_SCRATCH_BYTES = 32 << 20


class engram_config(ctypes.Structure):
    _fields_ = [
        ("n_orders", ctypes.c_int32),
        ("orders", ctypes.c_int32 * 4),
        ("heads", ctypes.c_int32),
        ("rows", ctypes.c_uint32 * ENGRAM_MAX_TABLES),
        ("mult", (ctypes.c_uint64 * 4) * ENGRAM_MAX_TABLES),
        ("row_dim", ctypes.c_int32),
        ("hidden", ctypes.c_int32),
        ("conv_width", ctypes.c_int32),
        ("vocab", ctypes.c_int32),
        ("canon_vocab", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("eps", ctypes.c_float),
    ]


class EngramError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.engram_strerror(status).decode()
        detail = _lib.engram_last_error().decode()
        super().__init__(f"{where}: {msg}" + (f" ({detail})" if detail else ""))


_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_st = ctypes.c_int
_sigs = {
    "engram_create": ([ctypes.POINTER(engram_config), ctypes.POINTER(_vp)], _st),
    "engram_destroy": ([_vp], None),
    "engram_strerror": ([_st], ctypes.c_char_p),
    "engram_last_error": ([], ctypes.c_char_p),
    "engram_workspace_bytes": ([_vp, _i32, _i32], _sz),
    "engram_profile_enable": ([_vp, _i32], _st),
    "engram_profile_read": ([_vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_char_p), _i32], _i32),
    "engram_device_status": ([_vp, _vp, ctypes.POINTER(ctypes.c_uint32)], _st),
    "engram_remap": ([_vp, _vp, _i64, _vp, _vp, _vp], _st),
    "engram_hash": ([_vp, _vp, _vp, _i32, _i32, _i64, _i32, _vp, _vp], _st),
    "engram_gather": ([_vp, _vp, _i64, _vp, _vp, _vp], _st),
    "engram_project": ([_vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp], _st),
    "engram_conv": ([_vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _i32, _vp], _st),
    "engram_gate_conv": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _sz, _vp],
                         _st),
    "engram_forward": ([_vp, _vp, _i32, _i32, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                        _i32, _vp, _sz, _vp], _st),
    "engram_forward_noalloc": ([_vp, _vp, _i32, _i32, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _vp, _i32, _vp], _st),
    "engram_host_workspace_bytes": ([_vp, _i32, _i32, _i32, _i32], _sz),
    "engram_host_tier_create": ([_vp, _vp, _i64, _i32, ctypes.POINTER(_vp)], _st),
    "engram_host_tier_destroy": ([_vp], None),
    "engram_host_dedupe": ([_vp, _vp, _i64, _vp], _st),
    "engram_host_fetch": ([_vp, _vp, ctypes.POINTER(_i64)], _st),
    "engram_gather_staged": ([_vp, _i64, _vp, _vp], _st),
    "engram_host_tier_stats": ([_vp, ctypes.c_void_p], _st),
    "engram_pack_rows": ([_vp, _i64, _sz, _vp, _i64, _vp, _i32], _st),
    "engram_debug_stall_next": ([_vp], _st),
    "engram_host_tier_debug": ([_vp, ctypes.c_uint32, ctypes.c_double], _st),
    "engram_host_cache_enable": ([_vp, _i64, _i32], _st),
    "engram_host_tier_map": ([_vp], _st),
    "engram_host_cache_reset": ([_vp, _vp], _st),
    "engram_host_cache_stats": ([_vp, ctypes.c_void_p], _st),
    "engram_shard_range": ([_vp, _i32, _i32, ctypes.POINTER(_i64), ctypes.POINTER(_i64)], _st),
    "engram_multibranch_workspace_bytes": ([_vp, _i32, _i32, _i32], _sz),
    "engram_table_grad_workspace_bytes": ([_vp, _i64], _sz),
    "engram_table_grad": ([_vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp], _st),
    "engram_table_sgd": ([_vp, _vp, _vp, _vp, _i64, _vp, ctypes.c_float, _vp], _st),
    "engram_grad_route_workspace_bytes": ([_vp], _sz),
    "engram_grad_route": ([_vp, _i32, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _sz, _vp], _st),
    "engram_grad_combine_workspace_bytes": ([_vp, _i64], _sz),
    "engram_grad_combine": ([_vp, _i32, _i32, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _sz, _vp], _st),
    "engram_shard_sgd": ([_vp, _i32, _i32, _vp, _vp, _vp, _i64, _vp, ctypes.c_float, _vp], _st),
    "engram_forward_multibranch": ([_vp, _i32, _vp, _i32, _i32, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                    _vp, _vp, _vp, _vp, _vp, _i32, _vp, _sz, _vp], _st),
    "engram_forward_sharded": ([_vp, _vp, _i32, _i32, _i64, _i32, _vp, ctypes.POINTER(_vp), _i32, _vp, _vp, _vp, _vp,
                                _vp, _vp, _vp, _vp, _vp, _i32, _vp, _sz, _vp], _st),
    "engram_ipc_export": ([_vp, _vp, ctypes.POINTER(ctypes.c_uint64)], _st),
    "engram_ipc_open": ([_vp, ctypes.c_uint64, ctypes.POINTER(_vp), ctypes.POINTER(_vp)], _st),
    "engram_ipc_close": ([_vp], _st),
    "engram_forward_host": ([_vp, _vp, _i32, _i32, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32,
                             _i32, _vp, _sz, _vp], _st),
}
for _name, (_args, _res) in _sigs.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res


def _ptr(t) -> Optional[int]:
    """Device pointer of a tensor (None for None)."""
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(status: int, where: str):
    if status != ENGRAM_OK:
        raise EngramError(status, where)


def make_config(orders: Sequence[int], heads: int, rows: Sequence[int], mult, row_dim: int, hidden: int,
                conv_width: int, vocab: int, canon_vocab: int, dtype: int, eps: float = 1e-6) -> engram_config:
    cfg = engram_config()
    cfg.n_orders = len(orders)
    for i, n in enumerate(orders):
        cfg.orders[i] = int(n)
    cfg.heads = heads
    for j, m in enumerate(rows):
        cfg.rows[j] = int(m)
    for j in range(len(rows)):
        for q in range(4):
            cfg.mult[j][q] = int(mult[j][q])
    cfg.row_dim, cfg.hidden, cfg.conv_width = row_dim, hidden, conv_width
    cfg.vocab, cfg.canon_vocab, cfg.dtype, cfg.eps = vocab, canon_vocab, dtype, eps
    return cfg


# ---------------------------------------------------------------- C ABI, same names

def engram_create(cfg: engram_config) -> int:
    ctx = _vp()
    _check(_lib.engram_create(ctypes.byref(cfg), ctypes.byref(ctx)), "engram_create")
    return ctx.value


def engram_destroy(ctx: int) -> None:
    _lib.engram_destroy(ctx)


def engram_strerror(status: int) -> str:
    return _lib.engram_strerror(status).decode()


def engram_last_error() -> str:
    return _lib.engram_last_error().decode()


def engram_workspace_bytes(ctx: int, B: int, L: int) -> int:
    return int(_lib.engram_workspace_bytes(ctx, B, L))


def engram_profile_enable(ctx: int, enable: bool = True) -> None:
    _check(_lib.engram_profile_enable(ctx, 1 if enable else 0), "engram_profile_enable")


def engram_profile_read(ctx: int, max_kernels: int = 16):
    """[(kernel name, ms)] of the kernels launched by the most recent call."""
    ms = (ctypes.c_float * max_kernels)()
    names = (ctypes.c_char_p * max_kernels)()
    n = _lib.engram_profile_read(ctx, ms, names, max_kernels)
    return [(names[i].decode(), float(ms[i])) for i in range(n)]


def engram_device_status(ctx: int, stream=None):
    """Returns (status, flags); does not raise."""
    flags = ctypes.c_uint32(0)
    st = _lib.engram_device_status(ctx, _stream(stream), ctypes.byref(flags))
    return int(st), int(flags.value)


def engram_remap(ctx, tok, n, P, canon, stream=None):
    _check(_lib.engram_remap(ctx, _ptr(tok), n, _ptr(P), _ptr(canon), _stream(stream)), "engram_remap")


def engram_hash(ctx, ids, P, B, T, stride, t_begin, idx, stream=None):
    _check(_lib.engram_hash(ctx, _ptr(ids), _ptr(P), B, T, stride, t_begin, _ptr(idx), _stream(stream)),
           "engram_hash")


def engram_gather(ctx, idx, n_tok, tables, e_cat, stream=None):
    _check(_lib.engram_gather(ctx, _ptr(idx), n_tok, _ptr(tables), _ptr(e_cat), _stream(stream)), "engram_gather")


def engram_project(ctx, e_cat, n_tok, h, Wk, Wv, gq, gk, v, part, stream=None):
    _check(_lib.engram_project(ctx, _ptr(e_cat), n_tok, _ptr(h), _ptr(Wk), _ptr(Wv), _ptr(gq), _ptr(gk), _ptr(v),
                               _ptr(part), _stream(stream)), "engram_project")


def engram_conv(ctx, v, part, h, conv_w, B, L, conv_state, y, alpha_out, add_residual, stream=None):
    _check(_lib.engram_conv(ctx, _ptr(v), _ptr(part), _ptr(h), _ptr(conv_w), B, L, _ptr(conv_state), _ptr(y),
                            _ptr(alpha_out), int(add_residual), _stream(stream)), "engram_conv")


def engram_gate_conv(ctx, e_cat, h, Wk, Wv, gq, gk, conv_w, B, L, conv_state, y, alpha_out, add_residual,
                     workspace, workspace_bytes, stream=None):
    _check(_lib.engram_gate_conv(ctx, _ptr(e_cat), _ptr(h), _ptr(Wk), _ptr(Wv), _ptr(gq), _ptr(gk), _ptr(conv_w),
                                 B, L, _ptr(conv_state), _ptr(y), _ptr(alpha_out), int(add_residual),
                                 _ptr(workspace), workspace_bytes, _stream(stream)), "engram_gate_conv")


def engram_forward(ctx, tok, B, T, tok_stride, t_begin, P, tables, h, Wk, Wv, gq, gk, conv_w, conv_state, y,
                   alpha_out, add_residual, workspace, workspace_bytes, stream=None):
    _check(_lib.engram_forward(ctx, _ptr(tok), B, T, tok_stride, t_begin, _ptr(P), _ptr(tables), _ptr(h), _ptr(Wk),
                               _ptr(Wv), _ptr(gq), _ptr(gk), _ptr(conv_w), _ptr(conv_state), _ptr(y),
                               _ptr(alpha_out), int(add_residual), _ptr(workspace), workspace_bytes,
                               _stream(stream)), "engram_forward")


def engram_forward_noalloc(ctx, tok, B, T, tok_stride, t_begin, P, tables, h, Wk, Wv, gq, gk, conv_w, conv_state, y,
                           alpha_out, add_residual, stream=None):
    """engram_forward with its scratch in the library's static device array
    (for callers that cannot allocate device memory)."""
    _check(_lib.engram_forward_noalloc(ctx, _ptr(tok), B, T, tok_stride, t_begin, _ptr(P), _ptr(tables), _ptr(h),
                                       _ptr(Wk), _ptr(Wv), _ptr(gq), _ptr(gk), _ptr(conv_w), _ptr(conv_state),
                                       _ptr(y), _ptr(alpha_out), int(add_residual), _stream(stream)),
           "engram_forward_noalloc")


def engram_host_workspace_bytes(ctx: int, B: int, T: int, t_begin: int, chunk_rows: int = 0) -> int:
    return int(_lib.engram_host_workspace_bytes(ctx, B, T, t_begin, chunk_rows))


def engram_forward_host(ctx, tok_host, B, T, tok_stride, t_begin, P, tables, h_host, Wk, Wv, gq, gk, conv_w,
                        conv_state, y_host, add_residual, chunk_rows, workspace, workspace_bytes, stream=None):
    """engram_forward with tok, h and y in host memory (CPU tensors, ideally
    pinned); the other tensors on the device."""
    _check(_lib.engram_forward_host(ctx, _ptr(tok_host), B, T, tok_stride, t_begin, _ptr(P), _ptr(tables),
                                    _ptr(h_host), _ptr(Wk), _ptr(Wv), _ptr(gq), _ptr(gk), _ptr(conv_w),
                                    _ptr(conv_state), _ptr(y_host), int(add_residual), chunk_rows, _ptr(workspace),
                                    workspace_bytes, _stream(stream)), "engram_forward_host")


# ---------------------------------------------------------------- multi-branch

def engram_multibranch_workspace_bytes(ctx, M: int, B: int, L: int) -> int:
    return int(_lib.engram_multibranch_workspace_bytes(ctx, M, B, L))


def engram_forward_multibranch(ctx, M, tok, B, T, tok_stride, t_begin, P, tables, h, Wk, Wv, gq, gk, k_scale,
                               v_scale, conv_w, conv_state, y, alpha_out, add_residual, workspace, workspace_bytes,
                               stream=None):
    _check(_lib.engram_forward_multibranch(ctx, M, _ptr(tok), B, T, tok_stride, t_begin, _ptr(P), _ptr(tables),
                                           _ptr(h), _ptr(Wk), _ptr(Wv), _ptr(gq), _ptr(gk), _ptr(k_scale),
                                           _ptr(v_scale), _ptr(conv_w),
                                           _ptr(conv_state), _ptr(y), _ptr(alpha_out), int(add_residual),
                                           _ptr(workspace), workspace_bytes, _stream(stream)),
           "engram_forward_multibranch")


# ---------------------------------------------------------------- table backward

def engram_table_grad_workspace_bytes(ctx, n_tok: int) -> int:
    return int(_lib.engram_table_grad_workspace_bytes(ctx, n_tok))


def engram_table_grad(ctx, idx, n_tok, d_e, rows_out, grad_out, n_unique, workspace, workspace_bytes, stream=None):
    _check(_lib.engram_table_grad(ctx, _ptr(idx), n_tok, _ptr(d_e), _ptr(rows_out), _ptr(grad_out), _ptr(n_unique),
                                  _ptr(workspace), workspace_bytes, _stream(stream)), "engram_table_grad")


def engram_table_sgd(ctx, rows, grad, n_unique, max_rows, tables, lr, stream=None):
    _check(_lib.engram_table_sgd(ctx, _ptr(rows), _ptr(grad), _ptr(n_unique), max_rows, _ptr(tables), float(lr),
                                 _stream(stream)), "engram_table_sgd")


def engram_grad_route_workspace_bytes(ctx) -> int:
    return int(_lib.engram_grad_route_workspace_bytes(ctx))


def engram_grad_route(ctx, n_shards, rows, grad, n_pairs, max_rows, send_rows, send_grad, send_counts, workspace,
                      workspace_bytes, stream=None):
    _check(_lib.engram_grad_route(ctx, n_shards, _ptr(rows), _ptr(grad), _ptr(n_pairs), max_rows, _ptr(send_rows),
                                  _ptr(send_grad), _ptr(send_counts), _ptr(workspace), workspace_bytes,
                                  _stream(stream)), "engram_grad_route")


def engram_grad_combine_workspace_bytes(ctx, n_pairs: int) -> int:
    return int(_lib.engram_grad_combine_workspace_bytes(ctx, n_pairs))


def engram_grad_combine(ctx, n_shards, shard, pair_rows, pair_grad, n_pairs, rows_out, grad_out, n_unique, workspace,
                        workspace_bytes, stream=None):
    _check(_lib.engram_grad_combine(ctx, n_shards, shard, _ptr(pair_rows), _ptr(pair_grad), n_pairs, _ptr(rows_out),
                                    _ptr(grad_out), _ptr(n_unique), _ptr(workspace), workspace_bytes,
                                    _stream(stream)), "engram_grad_combine")


def engram_shard_sgd(ctx, n_shards, shard, rows, grad, n_unique, max_rows, shard_table, lr, stream=None):
    _check(_lib.engram_shard_sgd(ctx, n_shards, shard, _ptr(rows), _ptr(grad), _ptr(n_unique), max_rows,
                                 _ptr(shard_table), float(lr), _stream(stream)), "engram_shard_sgd")


# ---------------------------------------------------------------- sharded tables

def engram_shard_range(ctx, n_shards: int, shard: int):
    """(first global row, row count) of shard `shard` of n_shards."""
    lo, cnt = _i64(0), _i64(0)
    _check(_lib.engram_shard_range(ctx, n_shards, shard, ctypes.byref(lo), ctypes.byref(cnt)), "engram_shard_range")
    return int(lo.value), int(cnt.value)


def engram_forward_sharded(ctx, tok, B, T, tok_stride, t_begin, P, shard_ptrs, h, Wk, Wv, gq, gk, conv_w,
                           conv_state, y, alpha_out, add_residual, workspace, workspace_bytes, stream=None):
    """shard_ptrs: device pointers (ints) of the shards, valid on the current device."""
    arr = (_vp * len(shard_ptrs))(*[int(p) if p else None for p in shard_ptrs])
    _check(_lib.engram_forward_sharded(ctx, _ptr(tok), B, T, tok_stride, t_begin, _ptr(P), arr, len(shard_ptrs),
                                       _ptr(h), _ptr(Wk), _ptr(Wv), _ptr(gq), _ptr(gk), _ptr(conv_w),
                                       _ptr(conv_state), _ptr(y), _ptr(alpha_out), int(add_residual),
                                       _ptr(workspace), workspace_bytes, _stream(stream)),
           "engram_forward_sharded")


def engram_ipc_export(dev_ptr: int):
    """(64-byte handle, offset) of the allocation holding dev_ptr."""
    buf = ctypes.create_string_buffer(ENGRAM_IPC_HANDLE_BYTES)
    off = ctypes.c_uint64(0)
    _check(_lib.engram_ipc_export(dev_ptr, buf, ctypes.byref(off)), "engram_ipc_export")
    return buf.raw, int(off.value)


def engram_ipc_open(handle: bytes, offset: int):
    """(pointer, mapping base) of an exported allocation, on the current device."""
    if len(handle) != ENGRAM_IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle is 64 bytes")
    ptr, base = _vp(), _vp()
    _check(_lib.engram_ipc_open(handle, offset, ctypes.byref(ptr), ctypes.byref(base)), "engram_ipc_open")
    return int(ptr.value), int(base.value)


def engram_ipc_close(base: int) -> None:
    _check(_lib.engram_ipc_close(base), "engram_ipc_close")


# ---------------------------------------------------------------- host tier

def engram_host_tier_create(ctx, host_tables, max_lookups: int, n_threads: int) -> int:
    """host_tables: a CPU tensor (or anything with data_ptr()) holding the
    [J][M][D] tables; it must outlive the tier."""
    out = _vp()
    _check(_lib.engram_host_tier_create(ctx, _ptr(host_tables), max_lookups, n_threads, ctypes.byref(out)),
           "engram_host_tier_create")
    return out.value


def engram_host_tier_debug(tier, inject: int, wait_limit_s: float) -> None:
    """Test hook: arm one-shot host-side faults of the next fetch and set the
    tier's host wait limit."""
    _check(_lib.engram_host_tier_debug(tier, inject, wait_limit_s), "engram_host_tier_debug")


def engram_host_tier_destroy(tier: int) -> None:
    _lib.engram_host_tier_destroy(tier)


def engram_host_dedupe(tier, idx, n_tok, stream=None):
    _check(_lib.engram_host_dedupe(tier, _ptr(idx), n_tok, _stream(stream)), "engram_host_dedupe")


def engram_host_fetch(tier, side_stream) -> int:
    n = _i64(0)
    _check(_lib.engram_host_fetch(tier, _stream(side_stream), ctypes.byref(n)), "engram_host_fetch")
    return int(n.value)


def engram_gather_staged(tier, n_tok, e_cat, stream=None):
    _check(_lib.engram_gather_staged(tier, n_tok, _ptr(e_cat), _stream(stream)), "engram_gather_staged")


class engram_host_tier_stats_t(ctypes.Structure):
    _fields_ = [("n_unique", ctypes.c_int64), ("n_copies", ctypes.c_int64), ("wait_ms", ctypes.c_double),
                ("pack_ms", ctypes.c_double), ("copy_ms", ctypes.c_double)]


def engram_host_tier_stats(tier) -> dict:
    """Figures of the last fetch: distinct rows, copies, host wait / packing
    ms, device copy ms (-1 while in flight)."""
    out = engram_host_tier_stats_t()
    _check(_lib.engram_host_tier_stats(tier, ctypes.addressof(out)), "engram_host_tier_stats")
    return {f: getattr(out, f) for f, _ in out._fields_}


def engram_host_tier_map(tier) -> None:
    """Map the host tables: the tier fetches rows with a GPU kernel over PCIe."""
    _check(_lib.engram_host_tier_map(tier), "engram_host_tier_map")


def engram_host_cache_enable(tier, capacity_rows: int, min_count: int = 2) -> None:
    _check(_lib.engram_host_cache_enable(tier, capacity_rows, min_count), "engram_host_cache_enable")


def engram_host_cache_reset(tier, stream=None) -> None:
    _check(_lib.engram_host_cache_reset(tier, _stream(stream)), "engram_host_cache_reset")


class engram_host_cache_stats_t(ctypes.Structure):
    _fields_ = [("capacity", ctypes.c_int64), ("resident", ctypes.c_int64), ("lookups", ctypes.c_int64),
                ("cached_lookups", ctypes.c_int64), ("cached_rows", ctypes.c_int64), ("fetched_rows", ctypes.c_int64)]


def engram_host_cache_stats(tier) -> dict:
    """Hot-row cache figures of the last batch."""
    out = engram_host_cache_stats_t()
    _check(_lib.engram_host_cache_stats(tier, ctypes.addressof(out)), "engram_host_cache_stats")
    return {f: getattr(out, f) for f, _ in out._fields_}


def engram_pack_rows(host_tables, total_rows: int, row_bytes: int, rows, n: int, dst, n_threads: int = 1):
    """Host-only packing: rows[i] of the tables into dst[i] (CPU tensors or numpy arrays)."""
    def addr(x):
        return x.ctypes.data if hasattr(x, "ctypes") else x.data_ptr()
    _check(_lib.engram_pack_rows(addr(host_tables), total_rows, row_bytes, addr(rows), n, addr(dst), n_threads),
           "engram_pack_rows")


def engram_debug_stall_next(ctx) -> None:
    """Test hook: the next fused key pass lets one bounded wait run out."""
    _check(_lib.engram_debug_stall_next(ctx), "engram_debug_stall_next")

"""Engram conditional-memory forward path for NVIDIA B200 (sm_100a).

The compute lives in ``libengram.so`` (CUDA kernels behind the C ABI declared
in ``include/engram.h``); :mod:`.binding` is its ctypes binding with the same
function names, and :class:`Engram` is a small convenience owner of a context
plus its workspace.  PyTorch is used only for device memory and streams.
"""

from __future__ import annotations

from typing import Optional

from .binding import (  # noqa: F401  (re-exported C ABI names)
    ENGRAM_BF16, ENGRAM_F32, ENGRAM_ERR_CANON, ENGRAM_ERR_INDEX, ENGRAM_ERR_TIMEOUT, ENGRAM_ERR_TOKEN,
    ENGRAM_E_CUDA, ENGRAM_E_DEVICE, ENGRAM_E_HOST, ENGRAM_E_INVAL, ENGRAM_E_NOMEM, ENGRAM_E_TIMEOUT,
    ENGRAM_E_UNSUPPORTED,
    ENGRAM_INVALID_INDEX, ENGRAM_OK, EXPORTS, LIB_PATH, EngramError, engram_config, engram_conv, engram_create,
    ENGRAM_NOALLOC_SCRATCH_BYTES, engram_destroy, engram_device_status, engram_forward, engram_forward_noalloc,
    engram_forward_host, engram_gate_conv, engram_gather, engram_gather_staged, engram_hash, engram_host_dedupe,
    engram_host_fetch, engram_host_tier_create, engram_host_tier_destroy, engram_host_tier_stats,
    engram_host_workspace_bytes, engram_pack_rows, engram_debug_stall_next,
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

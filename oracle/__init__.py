"""Engram forward oracle (TEST INFRASTRUCTURE ONLY).

Plain, single-threaded fp64 reference of the Engram forward path, in
``engram_oracle.cpp`` (built into ``liboracle.so`` by :func:`build`) with this
ctypes wrapper composing its steps in the order the pages give them
("DeepSeek AI II" digest, section "DeepSeek Engram"): remap, suffix n-grams,
multi-head hash, gather + concatenation, W_K / W_V projections, the scalar
gate, the causal depthwise convolution.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It shares no code with the CUDA library; the
only module both sides use is ``synth`` (seeded inputs, no method arithmetic).

Parity pins: every step is pinned by the CPU tests in ``tests/test_oracle_*.py``
(hand-derived golden cases, closed forms, invariants and library routines).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "engram_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", _LIB + ".tmp", _SRC]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def lib():
    """The loaded oracle library.  ``ORACLE_LIB`` names another build of
    ``engram_oracle.cpp`` (used only by the mutation test, which plants
    mistakes in a copy of the source to show that the pins catch them)."""
    global _lib
    if _lib is None:
        path = os.environ.get("ORACLE_LIB")
        if not path:
            path = build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        L.orc_remap.argtypes = [P, i64, P, i32, P]
        L.orc_remap.restype = i64
        L.orc_hash.argtypes = [P, i32, i32, i64, i32, i32, i32, P, i32, P, P, P]
        L.orc_hash.restype = i64
        L.orc_gather.argtypes = [P, i64, i32, P, P, i64, P]
        L.orc_gather.restype = None
        L.orc_project.argtypes = [P, i64, i32, P, i32, P]
        L.orc_project.restype = None
        L.orc_gate.argtypes = [P, P, i64, i32, P, P, f64, P]
        L.orc_gate.restype = None
        L.orc_conv.argtypes = [P, i32, i32, P, i32, P, P]
        L.orc_conv.restype = None
        L.orc_silu.argtypes = [f64]
        L.orc_silu.restype = f64
        L.orc_output.argtypes = [P, P, P, i64, i32, i32, P]
        L.orc_output.restype = None
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


# ---------------------------------------------------------------- steps

def remap(tok: np.ndarray, P: np.ndarray):
    """Step 1: canonical ids (-1 where the raw id is outside [0, V)); returns (canon, n_bad)."""
    tok = _c(tok, np.int32)
    P = _c(P, np.int32)
    canon = np.empty_like(tok)
    bad = lib().orc_remap(_p(tok), tok.size, _p(P), P.size, _p(canon))
    return canon, int(bad)


def hash_ids(canon: np.ndarray, Vc: int, orders, K: int, mult: np.ndarray, rows: np.ndarray,
             t_begin: int = 0):
    """Steps 2-3 over canon [B][T]: idx [B*(T-t_begin)][J] uint32; returns (idx, n_bad)."""
    canon = _c(canon, np.int32)
    B, T = canon.shape
    orders = _c(orders, np.int32)
    J = len(orders) * K
    mult = _c(mult, np.uint64).reshape(J, 4)
    rows = _c(rows, np.uint32)
    idx = np.empty((B * (T - t_begin), J), dtype=np.uint32)
    bad = lib().orc_hash(_p(canon), B, T, T, t_begin, Vc, len(orders), _p(orders), K,
                         _p(mult), _p(rows), _p(idx))
    return idx, int(bad)


def gather(idx: np.ndarray, rows: np.ndarray, tables: np.ndarray) -> np.ndarray:
    """Step 4 with host tables [J][M][D] (any element type): e_cat [n][J*D]."""
    idx = _c(idx, np.uint32)
    rows = _c(rows, np.uint32)
    tables = np.ascontiguousarray(tables)
    n, J = idx.shape
    D = tables.shape[-1]
    out = np.empty((n, J * D), dtype=tables.dtype)
    lib().orc_gather(_p(idx), n, J, _p(rows), _p(tables), D * tables.itemsize, _p(out))
    return out


def gather_rows(idx: np.ndarray, rows: np.ndarray, row_source) -> np.ndarray:
    """Step 4 where the tables are too large for the host: ``row_source(j, r)``
    returns the rows r of table j; rows are concatenated in table order
    (order ascending, head ascending).  An index >= M_j is a zero row."""
    idx = np.asarray(idx, dtype=np.uint32)
    n, J = idx.shape
    parts = []
    for j in range(J):
        r = idx[:, j].astype(np.int64)
        ok = r < int(rows[j])
        vals = row_source(j, np.where(ok, r, 0))
        vals = np.where(ok[:, None], vals, 0)
        parts.append(vals)
    return np.concatenate(parts, axis=1)


def project(e: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Step 5: e [n][d_mem] times W^T (W [d][d_mem]) in fp64."""
    e = _c(e, np.float64)
    W = _c(W, np.float64)
    n, dm = e.shape
    d = W.shape[0]
    out = np.empty((n, d), dtype=np.float64)
    lib().orc_project(_p(e), n, dm, _p(W), d, _p(out))
    return out


def gate(h: np.ndarray, k: np.ndarray, gq: np.ndarray, gk: np.ndarray, eps: float) -> np.ndarray:
    """Step 6: alpha [n]."""
    h = _c(h, np.float64)
    k = _c(k, np.float64)
    n, d = h.shape
    gq = _c(gq, np.float64)
    gk = _c(gk, np.float64)
    alpha = np.empty(n, dtype=np.float64)
    lib().orc_gate(_p(h), _p(k), n, d, _p(gq), _p(gk), float(eps), _p(alpha))
    return alpha


def conv(vt: np.ndarray, cw: np.ndarray, hist: Optional[np.ndarray] = None) -> np.ndarray:
    """Step 8 over one sequence segment vt [L][d]: u [L][d]."""
    vt = _c(vt, np.float64)
    L, d = vt.shape
    cw = _c(cw, np.float64)
    w = cw.shape[1]
    hist = None if hist is None else _c(hist, np.float64)
    u = np.empty_like(vt)
    lib().orc_conv(_p(vt), L, d, _p(cw), w, _p(hist), _p(u))
    return u


def output(vt: np.ndarray, u: np.ndarray, h: Optional[np.ndarray], add_residual: bool) -> np.ndarray:
    vt = _c(vt, np.float64)
    u = _c(u, np.float64)
    n, d = vt.shape
    hh = _c(h, np.float64) if add_residual else None
    y = np.empty_like(vt)
    lib().orc_output(_p(vt), _p(u), _p(hh), n, d, 1 if add_residual else 0, _p(y))
    return y


def silu(x: float) -> float:
    return lib().orc_silu(float(x))


# ---------------------------------------------------------------- composites

class Result:
    """Oracle outputs for a set of token rows."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def _value_path(e, h, Wk, Wv, gq, gk, eps):
    # k and v are kept at full precision: the pages fix no storage point for
    # them, and this build's rounding points are the stored tensors only
    # (tables/e, h, W, Y)
    k = project(e, Wk)
    v = project(e, Wv)
    alpha = gate(h, k, gq, gk, eps)
    return k, v, alpha


def forward_full(inp, add_residual: bool = False, eps: float = 1e-6, hist: Optional[np.ndarray] = None,
                 tables: Optional[np.ndarray] = None, h: Optional[np.ndarray] = None) -> Result:
    """Whole forward for a small workload (host tables); rows b-major."""
    wl = inp.wl
    canon, _ = remap(inp.tok, inp.P)
    idx, _ = hash_ids(canon, wl.Vc, wl.orders, wl.K, inp.mult, inp.rows, wl.t_begin)
    tables = inp.all_tables() if tables is None else tables
    e = gather(idx, inp.rows, tables)
    h = inp.all_hidden() if h is None else h
    k, v, alpha = _value_path(e, h, inp.Wk, inp.Wv, inp.gq, inp.gk, eps)
    vt = alpha[:, None] * v
    L = wl.T - wl.t_begin
    u = np.empty_like(vt)
    for b in range(wl.B):
        seg = slice(b * L, (b + 1) * L)
        u[seg] = conv(vt[seg], inp.conv_w, None if hist is None else hist[b])
    y = output(vt, u, h, add_residual)
    return Result(canon=canon, idx=idx, e=e, k=k, v=v, alpha=alpha, vt=vt, u=u, y=y)


def forward_rows(inp, positions: np.ndarray, add_residual: bool = False, eps: float = 1e-6,
                 hist: Optional[np.ndarray] = None, idx: Optional[np.ndarray] = None) -> Result:
    """Forward output at selected flat token rows, for workloads whose tables
    live on the device: each requested row needs its own and its w-1
    predecessors' gated values inside the same sequence; table and hidden rows
    are evaluated on the host from the seeded generator."""
    wl = inp.wl
    L = wl.T - wl.t_begin
    if idx is None:
        canon, _ = remap(inp.tok, inp.P)
        idx, _ = hash_ids(canon, wl.Vc, wl.orders, wl.K, inp.mult, inp.rows, wl.t_begin)
    need = set()
    for p in positions:
        b, t = divmod(int(p), L)
        for j in range(wl.w):
            if t - j >= 0:
                need.add(b * L + t - j)
    need = np.array(sorted(need), dtype=np.int64)
    slot = {int(r): i for i, r in enumerate(need)}
    e = gather_rows(idx[need], inp.rows, inp.table_rows)
    h = inp.hidden_rows(need)
    k, v, alpha = _value_path(e, h, inp.Wk, inp.Wv, inp.gq, inp.gk, eps)
    vt = alpha[:, None] * v
    y = np.empty((len(positions), wl.d))
    al = np.empty(len(positions))
    win = np.zeros((len(positions), wl.w, wl.d))
    for i, p in enumerate(positions):
        b, t = divmod(int(p), L)
        lo = max(0, t - (wl.w - 1))
        seg = np.stack([vt[slot[b * L + tt]] for tt in range(lo, t + 1)])
        if lo == 0 and hist is not None:
            u = conv(seg, inp.conv_w, hist[b])[-1:]
        else:
            u = conv(seg, inp.conv_w, None)[-1:]
        y[i] = output(vt[slot[int(p)]][None], u, h[slot[int(p)]][None], add_residual)[0]
        al[i] = alpha[slot[int(p)]]
        for j in range(wl.w):
            if t - j >= 0:
                win[i, j] = vt[slot[b * L + t - j]]
            elif hist is not None:
                win[i, j] = hist[b][wl.w - 1 + t - j]
    return Result(idx=idx, y=y, alpha=al, vt_win=win, positions=np.asarray(positions))


def vt_windows(vt: np.ndarray, B: int, L: int, w: int, hist: Optional[np.ndarray] = None) -> np.ndarray:
    """[n][w][d]: the gated values v~_{t-j}, j < w, seen by each row's conv."""
    n, d = vt.shape
    win = np.zeros((n, w, d))
    for r in range(n):
        b, t = divmod(r, L)
        for j in range(w):
            if t - j >= 0:
                win[r, j] = vt[b * L + t - j]
            elif hist is not None:
                win[r, j] = hist[b][w - 1 + t - j]
    return win


def forward_multibranch(branches, add_residual: bool = False, eps: float = 1e-6,
                        hist: Optional[np.ndarray] = None, tables: Optional[np.ndarray] = None,
                        h: Optional[np.ndarray] = None) -> Result:
    """Multi-branch Engram ("DeepSeek AI II" digest, section "DeepSeek
    Engram", the multi-branch paragraphs): the M branches share the tables
    and W_V, branch m has its own W_K^(m), hidden state h^(m) and gate
    alpha^(m) = sigmoid(<RMSNorm(h^(m)), RMSNorm(W_K^(m) e)> / sqrt(d)), and
    u^(m) = alpha^(m) * (W_V e).  Each branch's gated value then goes through
    the single-branch conv and output (shared taps, a history per branch).

    branches[m] holds branch m's W_K, gains and hidden rows; branches[0] also
    the shared tokens, tables, W_V and conv taps.  hist: [M][B][w-1][d] or
    None; h: [M][n][d] or None (then each branch's all_hidden())."""
    inp = branches[0]
    wl = inp.wl
    M = len(branches)
    canon, _ = remap(inp.tok, inp.P)
    idx, _ = hash_ids(canon, wl.Vc, wl.orders, wl.K, inp.mult, inp.rows, wl.t_begin)
    tables = inp.all_tables() if tables is None else tables
    e = gather(idx, inp.rows, tables)
    v = project(e, inp.Wv)
    L = wl.T - wl.t_begin
    ys, alphas, vts = [], [], []
    for m, br in enumerate(branches):
        hm = br.all_hidden() if h is None else h[m]
        k = project(e, br.Wk)
        alpha = gate(hm, k, br.gq, br.gk, eps)
        vt = alpha[:, None] * v
        u = np.empty_like(vt)
        for b in range(wl.B):
            seg = slice(b * L, (b + 1) * L)
            u[seg] = conv(vt[seg], inp.conv_w, None if hist is None else hist[m][b])
        ys.append(output(vt, u, hm, add_residual))
        alphas.append(alpha)
        vts.append(vt)
    return Result(idx=idx, e=e, v=v, alpha=np.stack(alphas), vt=np.stack(vts), y=np.stack(ys))


def table_grad(idx: np.ndarray, rows: np.ndarray, de: np.ndarray, D: int):
    """Gradient of the tables from dL/de ("DeepSeek AI II" digest, section
    "DeepSeek Engram", training): e_t concatenates E_j[idx_j(t)], so the
    gradient of table j's row r is the sum of slice j of dL/de_t over the
    lookups with idx_j(t) = r.  Returns (sorted distinct global rows
    sum_{i<j} M_i + r, fp64 [U][D] gradients); invalid indices contribute
    nothing."""
    idx = np.asarray(idx, dtype=np.uint32)
    n, J = idx.shape
    de = np.asarray(de, dtype=np.float64).reshape(n, J, D)
    off = np.concatenate([[0], np.cumsum(np.asarray(rows, dtype=np.int64)[:-1])])
    r = idx.astype(np.int64)
    valid = r < np.asarray(rows, dtype=np.int64)[None, :]
    keys = (r + off[None, :])[valid]
    uniq, inv = np.unique(keys, return_inverse=True)
    grad = np.zeros((len(uniq), D))
    np.add.at(grad, inv, de[valid])
    return uniq, grad


def decode_e4m3(codes) -> np.ndarray:
    """Values of FP8 E4M3 codes, from the format's definition (OCP 8-bit
    floating point, E4M3): bit 7 the sign, bits 6-3 the exponent with bias 7,
    bits 2-0 the mantissa; exponent 0 holds the subnormals m/8 * 2^-6; the
    code with exponent 15 and mantissa 7 is NaN; there are no infinities
    (largest finite value 448).  The tables and weights of the FP8 path are
    such codes ("DeepSeek AI II" digest, section "DeepSeek Engram": the fused
    projections run as one dense FP8 GEMM)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    mag = np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)
    return sign * mag

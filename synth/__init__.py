"""Seeded synthetic inputs for the Engram forward path.

This module is shared by the oracle side (``oracle/``, ``tests/``) and the
device side (``bench.py``, the GPU tests).  It holds none of the method's
arithmetic: it only draws token streams, the compression surjection, the hash
multipliers and the floating-point tensors (tables, hidden states, weights).

Everything is a pure function of a workload's seed:

* token ids are i.i.d. Zipf over the raw vocabulary (the pages say natural
  n-grams are Zipfian; DeepSeek Engram digest, "system efficiency" section),
  drawn with numpy's PCG64 by inverse CDF;
* the compression map P is a seeded surjection V -> V' (the pages' tokenizer
  compression; the real map needs the DeepSeek-V3 vocabulary, which is not
  available, so a random surjection of the same sizes stands in for it);
* the hash multipliers a_{n,k,j} are consecutive outputs of SplitMix64
  (Steele, Lea and Flood, OOPSLA 2014) from a fixed seed, forced odd;
* every floating-point tensor element is a counter-based value: element i of
  stream ``key`` is SplitMix64's mixing function applied to
  ``key + (i + 1) * 0x9E3779B97F4A7C15`` (the i-th output of a SplitMix64
  generator seeded with ``key``), whose four 16-bit chunks are summed
  (Irwin-Hall of order 4) and centred/scaled to unit variance.  The result
  approximates N(0, 1) with tails capped at +-3.46 sigma.  The same element
  can be produced by numpy on the host or by torch integer ops on the GPU, so
  the oracle can evaluate any row of a 37 GB device table without copying it.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Sequence

import numpy as np

GOLDEN = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB
MASK64 = (1 << 64) - 1
HASH_SEED = 0x454E4752414D  # ASCII "ENGRAM"

# Irwin-Hall(4) of 16-bit chunks: sum of four discrete uniforms on [0, 65535].
_IH_MEAN = 4 * 32767.5
_IH_SD = math.sqrt(4.0 * (65536.0 ** 2 - 1.0) / 12.0)

# stream tags for the float tensors
TAG_TABLES, TAG_HIDDEN, TAG_WK, TAG_WV, TAG_CONV, TAG_GQ, TAG_GK, TAG_STATE = range(1, 9)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: sizes, distributions and seed."""

    name: str
    B: int                 # sequences
    T: int                 # positions per sequence seen so far
    t_begin: int           # first position computed (0: prefill, T-1: decode)
    V: int                 # raw vocabulary
    Vc: int                # canonical vocabulary V' (PAD id = Vc)
    zipf_s: float
    orders: tuple
    K: int                 # hash heads per order
    M: int                 # rows per table (prime)
    D: int                 # row width
    d: int                 # hidden width
    w: int                 # conv kernel width
    dtype: str             # "f32" or "bf16"
    seed: int
    table_sd: float = 0.02
    host_tables: bool = False

    @property
    def J(self) -> int:
        return len(self.orders) * self.K

    @property
    def d_mem(self) -> int:
        return self.J * self.D

    @property
    def n_tok(self) -> int:
        return self.B * (self.T - self.t_begin)

    @property
    def elem_bytes(self) -> int:
        """bytes of a table element (h and Y are bf16 for "bf16" and "fp8")"""
        return {"f32": 4, "bf16": 2, "fp8": 1}[self.dtype]

    @property
    def w_sd(self) -> float:
        # W ~ N(0, sigma_W^2) with sigma_W = 1 / (4 sigma_E sqrt(d_mem)), so that
        # k and v have standard deviation 0.25 (keeps |Y| = O(1)).
        return 1.0 / (4.0 * self.table_sd * math.sqrt(self.d_mem))

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    # tiny, CPU-checkable: 4096 -> 3154 ids, K=2, 4 tables of 10007 x 32 fp32
    "c1": Workload("c1", B=1, T=256, t_begin=0, V=4096, Vc=3154, zipf_s=1.1,
                   orders=(2, 3), K=2, M=10007, D=32, d=256, w=4, dtype="f32", seed=0),
    # 16 tables x 1000003 x 64 bf16 (~2 GB), d_mem 1024, d 2560
    "c2": Workload("c2", B=4, T=4096, t_begin=0, V=128000, Vc=98560, zipf_s=1.1,
                   orders=(2, 3), K=8, M=1000003, D=64, d=2560, w=4, dtype="bf16", seed=1),
    # 27B-style: 16 tables x 2781271 x 128 bf16 (11.4 GB), d_mem 2048
    "c3": Workload("c3", B=8, T=4096, t_begin=0, V=128000, Vc=98560, zipf_s=1.1,
                   orders=(2, 3), K=8, M=2781271, D=128, d=2560, w=4, dtype="bf16", seed=2),
    # 40B-style decode: 256 sequences, 8191 context + 1 new token; 9030011 is
    # not prime, the next prime 9030017 is used (37 GB of tables)
    "c4": Workload("c4", B=256, T=8192, t_begin=8191, V=128000, Vc=98560, zipf_s=1.0,
                   orders=(2, 3), K=8, M=9030017, D=128, d=2560, w=4, dtype="bf16", seed=3),
    # host-memory tier: 48828127 is not prime, 48828139 is; the row count is
    # scaled down to fit host RAM by the host-tier tests and bench
    "c5": Workload("c5", B=8, T=4096, t_begin=0, V=128000, Vc=98560, zipf_s=1.1,
                   orders=(2, 3), K=8, M=48828139, D=128, d=2560, w=4, dtype="bf16", seed=4,
                   host_tables=True),
}


# FP8 (E4M3) inputs: the tables are stored as E4M3 codes of value / FP8_TABLE_SCALE
# (the Irwin-Hall tails, 3.46 sigma, stay below the format's largest value, 448),
# each weight row as E4M3 codes of W[c] / s_W[c] with s_W[c] = max |W[c]| / 448.
FP8_MAX = 448.0


def fp8_table_scale(wl: "Workload") -> float:
    return float(np.float32(3.5 * wl.table_sd / FP8_MAX))


def fp8_codes(x: np.ndarray) -> np.ndarray:
    """uint8 E4M3 codes of fp32 values (torch's round-to-nearest conversion)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def fp8_values(codes: np.ndarray) -> np.ndarray:
    """fp32 values of E4M3 codes (torch's conversion)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).to(torch.float32).numpy()


def _is_prime(n: int) -> bool:
    if n < 2:
        return False
    if n % 2 == 0:
        return n == 2
    f = 3
    while f * f <= n:
        if n % f == 0:
            return False
        f += 2
    return True


def host_scaled(wl: Workload, mem_bytes: int) -> Workload:
    """The host-memory workload with its tables shrunk to fit ``mem_bytes``:
    rows per table = the largest prime not above the stated size whose
    J x rows x D tables fit (the sizing rule for a box with less host memory
    than the stated 200 GB)."""
    per_row = wl.J * wl.D * wl.elem_bytes
    m = min(wl.M, int(mem_bytes // per_row))
    while m > 2 and not _is_prime(m):
        m -= 1
    return wl if m == wl.M else wl.replace(M=m)


def workload(name_or_wl) -> Workload:
    if isinstance(name_or_wl, Workload):
        return name_or_wl
    return WORKLOADS[name_or_wl]


# ---------------------------------------------------------------- SplitMix64

def splitmix64_stream(seed: int, count: int) -> list:
    """The first ``count`` outputs of SplitMix64 seeded with ``seed`` (Python ints)."""
    out = []
    x = seed & MASK64
    for _ in range(count):
        x = (x + GOLDEN) & MASK64
        z = x
        z = ((z ^ (z >> 30)) * MIX1) & MASK64
        z = ((z ^ (z >> 27)) * MIX2) & MASK64
        out.append(z ^ (z >> 31))
    return out


def _stream_key(seed: int, tag: int) -> int:
    return splitmix64_stream((seed << 8) | tag, 1)[0]


def _mix_np(x: np.ndarray) -> np.ndarray:
    z = x
    z = (z ^ (z >> np.uint64(30))) * np.uint64(MIX1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(MIX2)
    return z ^ (z >> np.uint64(31))


def _ih_to_f32(z: np.ndarray, scale: float) -> np.ndarray:
    m = np.uint64(0xFFFF)
    s = ((z & m) + ((z >> np.uint64(16)) & m) + ((z >> np.uint64(32)) & m)
         + (z >> np.uint64(48))).astype(np.int64)
    # (S - mean) * 2 is an exact integer; one fp32 multiply by a fp32 constant
    centred2 = (2 * s - int(2 * _IH_MEAN)).astype(np.float32)
    return centred2 * np.float32(scale / (2.0 * _IH_SD))


def normal_np(seed: int, tag: int, flat_index: np.ndarray, scale: float) -> np.ndarray:
    """Counter-based approximately-normal fp32 values at the given flat indices."""
    key = np.uint64(_stream_key(seed, tag))
    i = np.asarray(flat_index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        x = key + (i + np.uint64(1)) * np.uint64(GOLDEN)
        return _ih_to_f32(_mix_np(x), scale)


def _s64(v: int) -> int:
    v &= MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def normal_torch(seed: int, tag: int, start: int, n: int, scale: float, device):
    """Same values as :func:`normal_np` for flat indices [start, start+n), built
    with torch int64 ops on ``device`` (two's-complement wrap-around)."""
    import torch
    key = _stream_key(seed, tag)
    i = torch.arange(start + 1, start + n + 1, dtype=torch.int64, device=device)
    x = i * _s64(GOLDEN) + _s64(key)

    def lsr(t, s):
        return (t >> s) & ((1 << (64 - s)) - 1)

    z = (x ^ lsr(x, 30)) * _s64(MIX1)
    z = (z ^ lsr(z, 27)) * _s64(MIX2)
    z = z ^ lsr(z, 31)
    del x, i
    s = (z & 0xFFFF) + (lsr(z, 16) & 0xFFFF) + (lsr(z, 32) & 0xFFFF) + lsr(z, 48)
    del z
    centred2 = (2 * s - int(2 * _IH_MEAN)).to(torch.float32)
    return centred2 * float(np.float32(scale / (2.0 * _IH_SD)))


# ---------------------------------------------------------------- token streams

def zipf_tokens(wl: Workload, B: Optional[int] = None, T: Optional[int] = None) -> np.ndarray:
    """int32 [B][T] token ids, P(id = r-1) proportional to r^-s, r in [1, V]."""
    B = wl.B if B is None else B
    T = wl.T if T is None else T
    rng = np.random.Generator(np.random.PCG64(wl.seed * 7919 + 17))
    r = np.arange(1, wl.V + 1, dtype=np.float64)
    p = r ** (-wl.zipf_s)
    cdf = np.cumsum(p)
    cdf /= cdf[-1]
    u = rng.random(B * T)
    ids = np.searchsorted(cdf, u, side="right")
    return np.minimum(ids, wl.V - 1).astype(np.int32).reshape(B, T)


def surjection(wl: Workload) -> np.ndarray:
    """int32 [V] map onto [0, V'): a seeded permutation pi with P(pi(j)) = j for
    j < V', the remaining V - V' raw ids sent uniformly into [0, V')."""
    rng = np.random.Generator(np.random.PCG64(wl.seed * 7919 + 29))
    pi = rng.permutation(wl.V)
    P = np.empty(wl.V, dtype=np.int32)
    P[pi[: wl.Vc]] = np.arange(wl.Vc, dtype=np.int32)
    P[pi[wl.Vc:]] = rng.integers(0, wl.Vc, size=wl.V - wl.Vc, dtype=np.int32)
    return P


def hash_multipliers(wl: Workload, seed: int = HASH_SEED) -> np.ndarray:
    """uint64 [J][4]: a_{n,k,j} for table (order o, head k) at row o*K + k, drawn
    as consecutive SplitMix64 outputs in (order, head, j) order, forced odd;
    entries j >= n are zero."""
    J = wl.J
    need = sum(n * wl.K for n in wl.orders)
    stream = iter(splitmix64_stream(seed, need))
    a = np.zeros((J, 4), dtype=np.uint64)
    for o, n in enumerate(wl.orders):
        for k in range(wl.K):
            for j in range(n):
                a[o * wl.K + k, j] = next(stream) | 1
    return a


def table_rows_np(wl: Workload, j: int, rows: np.ndarray, M: Optional[int] = None) -> np.ndarray:
    """fp32 [len(rows)][D] values of table j (before any bf16 rounding)."""
    M = wl.M if M is None else M
    rows = np.asarray(rows, dtype=np.int64)
    base = (j * M + rows)[:, None] * wl.D + np.arange(wl.D, dtype=np.int64)[None, :]
    return normal_np(wl.seed, TAG_TABLES, base.reshape(-1), wl.table_sd).reshape(len(rows), wl.D)


# ---------------------------------------------------------------- input bundle

class Inputs:
    """All inputs of one workload.  Small float tensors are kept as host numpy
    arrays (fp32 values; bf16 workloads store the bf16-rounded values as
    uint16 bit patterns in ``*_bits``); tensors that live on a device are
    built there by :meth:`to_device`."""

    def __init__(self, wl: Workload, gamma: str = "ones", M: Optional[int] = None,
                 B: Optional[int] = None):
        wl = wl if B is None else wl.replace(B=B)
        self.wl = wl
        self.M = wl.M if M is None else M
        self.tok = zipf_tokens(wl)
        self.P = surjection(wl)
        self.mult = hash_multipliers(wl)
        self.rows = np.full(wl.J, self.M, dtype=np.uint32)
        d, dm = wl.d, wl.d_mem
        self.Wk = normal_np(wl.seed, TAG_WK, np.arange(d * dm), wl.w_sd).reshape(d, dm)
        self.Wv = normal_np(wl.seed, TAG_WV, np.arange(d * dm), wl.w_sd).reshape(d, dm)
        self.conv_w = normal_np(wl.seed, TAG_CONV, np.arange(d * wl.w),
                                1.0 / math.sqrt(wl.w)).reshape(d, wl.w)
        if gamma == "ones":
            self.gq = np.ones(d, dtype=np.float32)
            self.gk = np.ones(d, dtype=np.float32)
        else:
            # positive gains in [0.5, 1.5]
            self.gq = (1.0 + 0.5 * np.tanh(normal_np(wl.seed, TAG_GQ, np.arange(d), 1.0))).astype(np.float32)
            self.gk = (1.0 + 0.5 * np.tanh(normal_np(wl.seed, TAG_GK, np.arange(d), 1.0))).astype(np.float32)
        if wl.dtype == "bf16":
            self.Wk = to_bf16_values(self.Wk)
            self.Wv = to_bf16_values(self.Wv)
        self.k_scale = self.v_scale = None
        if wl.dtype == "fp8":
            # codes per row, and the per-channel scale the GEMM epilogue applies:
            # table scale x row scale; Wk / Wv hold scale[c] * decoded codes, so that
            # W e over the decoded table values is the device's k and v
            te = fp8_table_scale(wl)
            self.Wk_codes, self.k_scale = self._fp8_rows(self.Wk, te)
            self.Wv_codes, self.v_scale = self._fp8_rows(self.Wv, te)
            self.Wk = self.k_scale.astype(np.float64)[:, None] * fp8_values(self.Wk_codes).astype(np.float64)
            self.Wv = self.v_scale.astype(np.float64)[:, None] * fp8_values(self.Wv_codes).astype(np.float64)

    @staticmethod
    def _fp8_rows(W: np.ndarray, table_scale: float):
        W = np.asarray(W, dtype=np.float32)
        s_w = (np.max(np.abs(W), axis=1) / np.float32(FP8_MAX)).astype(np.float32)
        codes = fp8_codes(W / s_w[:, None])
        return codes, (s_w * np.float32(table_scale)).astype(np.float32)

    # -- rows of the big tensors, computed on the host on demand
    def table_rows(self, j: int, rows: np.ndarray) -> np.ndarray:
        """Table values as the path sees them: bf16-rounded, or, for FP8, the
        decoded E4M3 values (the table scale is in k_scale / v_scale)."""
        v = table_rows_np(self.wl, j, rows, self.M)
        if self.wl.dtype == "fp8":
            return fp8_values(fp8_codes(v / np.float32(fp8_table_scale(self.wl))))
        return to_bf16_values(v) if self.wl.dtype == "bf16" else v

    def hidden_rows(self, rows: np.ndarray) -> np.ndarray:
        """h rows (flat token-row index in [0, n_tok)), N(0, 1)."""
        rows = np.asarray(rows, dtype=np.int64)
        d = self.wl.d
        base = rows[:, None] * d + np.arange(d, dtype=np.int64)[None, :]
        v = normal_np(self.wl.seed, TAG_HIDDEN, base.reshape(-1), 1.0).reshape(len(rows), d)
        return v if self.wl.dtype == "f32" else to_bf16_values(v)

    def state_rows(self, b: np.ndarray) -> np.ndarray:
        """Conv history [len(b)][w-1][d] fp32 used by decode tests (scale 0.25)."""
        b = np.asarray(b, dtype=np.int64)
        n = (self.wl.w - 1) * self.wl.d
        base = b[:, None] * n + np.arange(n, dtype=np.int64)[None, :]
        return normal_np(self.wl.seed, TAG_STATE, base.reshape(-1), 0.25).reshape(len(b), self.wl.w - 1, self.wl.d)

    def all_tables(self) -> np.ndarray:
        """[J][M][D] fp32 values (small workloads only; FP8: the decoded codes)."""
        wl = self.wl
        out = np.empty((wl.J, self.M, wl.D), dtype=np.float32)
        for j in range(wl.J):
            out[j] = self.table_rows(j, np.arange(self.M))
        return out

    def all_hidden(self) -> np.ndarray:
        return self.hidden_rows(np.arange(self.wl.n_tok))

    # -- device tensors (torch); tables and h generated on the device
    def _table_dtype(self):
        import torch
        return {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.uint8}[self.wl.dtype]

    def _to_table(self, x):
        """fp32 generator values -> the stored table element (FP8: E4M3 codes)"""
        import torch
        if self.wl.dtype == "fp8":
            return (x / float(np.float32(fp8_table_scale(self.wl)))).to(torch.float8_e4m3fn).view(torch.uint8)
        return x.to(self._table_dtype())

    def device_tables(self, device, chunk: int = 1 << 27):
        import torch
        wl = self.wl
        n = wl.J * self.M * wl.D
        out = torch.empty(n, dtype=self._table_dtype(), device=device)
        for s in range(0, n, chunk):
            e = min(n, s + chunk)
            out[s:e] = self._to_table(normal_torch(wl.seed, TAG_TABLES, s, e - s, wl.table_sd, device))
        return out.view(wl.J, self.M, wl.D)

    def device_table_range(self, first_row: int, n_rows: int, out, chunk: int = 1 << 27):
        """Rows [first_row, first_row + n_rows) of the J tables numbered back to
        back (table j's row r is row j * M + r) into ``out`` ([n_rows][D] on a
        device): the same values as device_tables, for one shard of them."""
        wl = self.wl
        flat = out.view(-1)
        n = n_rows * wl.D
        for s in range(0, n, chunk):
            e = min(n, s + chunk)
            flat[s:e] = self._to_table(normal_torch(wl.seed, TAG_TABLES, first_row * wl.D + s, e - s, wl.table_sd,
                                                    out.device))
        return out

    def host_tables(self, device, chunk: int = 1 << 27, pin: bool = False):
        """[J][M][D] tables in host memory (torch CPU tensor), the same values
        as device_tables: generated on ``device`` in chunks and copied out."""
        import torch
        wl = self.wl
        n = wl.J * self.M * wl.D
        out = torch.empty(n, dtype=self._table_dtype(), pin_memory=pin)
        for s in range(0, n, chunk):
            e = min(n, s + chunk)
            out[s:e].copy_(self._to_table(normal_torch(wl.seed, TAG_TABLES, s, e - s, wl.table_sd, device)))
        return out.view(wl.J, self.M, wl.D)

    def device_hidden(self, device, chunk: int = 1 << 27):
        import torch
        wl = self.wl
        n = wl.n_tok * wl.d
        tdt = torch.float32 if wl.dtype == "f32" else torch.bfloat16     # h: bf16 for bf16 and FP8
        out = torch.empty(n, dtype=tdt, device=device)
        for s in range(0, n, chunk):
            e = min(n, s + chunk)
            out[s:e] = normal_torch(wl.seed, TAG_HIDDEN, s, e - s, 1.0, device).to(tdt)
        return out.view(wl.n_tok, wl.d)

    def device_state(self, device):
        import torch
        wl = self.wl
        n = wl.B * (wl.w - 1) * wl.d
        return normal_torch(wl.seed, TAG_STATE, 0, n, 0.25, device).view(wl.B, wl.w - 1, wl.d)

    def device_dense(self, device):
        """dict of small device tensors: tok, P, Wk, Wv, conv_w, gq, gk (and, for
        FP8, Wk/Wv as E4M3 codes plus k_scale, v_scale)."""
        import torch
        tdt = torch.float32 if self.wl.dtype == "f32" else torch.bfloat16
        if self.wl.dtype == "fp8":
            w = {"Wk": torch.from_numpy(self.Wk_codes).to(device), "Wv": torch.from_numpy(self.Wv_codes).to(device),
                 "k_scale": torch.from_numpy(self.k_scale).to(device),
                 "v_scale": torch.from_numpy(self.v_scale).to(device)}
        else:
            w = {"Wk": torch.from_numpy(self.Wk).to(tdt).to(device), "Wv": torch.from_numpy(self.Wv).to(tdt).to(device),
                 "k_scale": None, "v_scale": None}
        return {
            "tok": torch.from_numpy(self.tok).to(device),
            "P": torch.from_numpy(self.P).to(device),
            **w,
            "conv_w": torch.from_numpy(self.conv_w).to(device),
            "gq": torch.from_numpy(self.gq).to(device),
            "gk": torch.from_numpy(self.gk).to(device),
        }


def branch_inputs(inp: "Inputs", m: int, gamma: str = "random") -> "Inputs":
    """Inputs of branch m of a multi-branch module: its own key projection,
    RMSNorm gains and hidden states, drawn from a seed of their own; branch 0
    is ``inp`` itself.  The tokens, tables, W_V and conv taps of the module
    are branch 0's (the caller uses those of ``inp``)."""
    if m == 0:
        return inp
    return Inputs(inp.wl.replace(seed=inp.wl.seed * 31 + 977 * m), gamma=gamma, M=inp.M)


def to_bf16_values(x: np.ndarray) -> np.ndarray:
    """fp32 values rounded to the nearest bf16 (ties to even), returned as fp32."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of fp32 values that are already bf16-representable."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    assert not np.any(b & 0xFFFF), "values are not bf16-representable"
    return (b >> 16).astype(np.uint16)


def sample_positions(wl: Workload, n: int, seed: int = 0) -> np.ndarray:
    """Flat token-row indices (b * (T - t_begin) + t - t_begin) for sampled
    parity: every sequence's first four and last computed positions plus
    uniformly drawn ones."""
    L = wl.T - wl.t_begin
    pick = set()
    for b in range(wl.B):
        for t in list(range(min(L, 4))) + [L - 1]:
            pick.add(b * L + t)
    rng = np.random.Generator(np.random.PCG64(seed + 991))
    extra = rng.integers(0, wl.n_tok, size=max(0, n - len(pick)))
    pick.update(int(x) for x in extra)
    return np.array(sorted(pick), dtype=np.int64)

"""Helpers shared by the GPU parity tests: build a context from seeded inputs,
place the inputs on the device, and the bf16 output tolerance."""

from __future__ import annotations

import numpy as np

import synth


def config_for(inp, eb, eps: float = 1e-6):
    wl = inp.wl
    return eb.make_config(orders=wl.orders, heads=wl.K, rows=[int(x) for x in inp.rows], mult=inp.mult,
                          row_dim=wl.D, hidden=wl.d, conv_width=wl.w, vocab=wl.V, canon_vocab=wl.Vc,
                          dtype={"bf16": eb.ENGRAM_BF16, "f32": eb.ENGRAM_F32, "fp8": eb.ENGRAM_FP8}[wl.dtype], eps=eps)


class DeviceInputs:
    def __init__(self, inp, device="cuda:0"):
        import torch
        self.inp = inp
        self.wl = inp.wl
        dd = inp.device_dense(device)
        self.__dict__.update(dd)
        self.tables = inp.device_tables(device)
        self.h = inp.device_hidden(device)
        self.dtype = torch.float32 if self.wl.dtype == "f32" else torch.bfloat16
        self.device = device

    def empty_y(self):
        import torch
        return torch.empty(self.wl.n_tok, self.wl.d, dtype=self.dtype, device=self.device)


def bf16_bound(y_ref: np.ndarray, vt_win: np.ndarray, cw: np.ndarray) -> np.ndarray:
    """Elementwise bound on |Y_gpu - Y_oracle| for the bf16 path.

    Sources: (1) Y is rounded once to bf16 (half an ulp, 2^-8 relative);
    (2) the fused epilogue evaluates the tap sum in fp32 and SiLU through the
    hardware tanh approximation (relative error about 2^-11), both far under
    2^-8 of sum_j |c_j| |v~_{t-j}|.  The accumulation order of v (fp32)
    differs from the oracle's (fp64) only in the last bits.  An error of
    relative size r in v~_{t-j} reaches Y_t through the skip (j = 0, weight 1)
    and through SiLU(u) (weight |c_j| * max SiLU', max SiLU' < 1.1).  The
    bound allows r = 2^-7 per term and a factor 1.5 on the sum; (3) fp32
    arithmetic in the gate and the skip/residual add stays well below 1e-5
    at these magnitudes."""
    w = cw.shape[1]
    s = np.abs(vt_win[:, 0]) * (1.0 + 1.1 * np.abs(cw[None, :, 0]))
    for j in range(1, w):
        s = s + 1.1 * np.abs(cw[None, :, j]) * np.abs(vt_win[:, j])
    return 1.5 * (2.0 ** -8 * np.abs(y_ref) + 2.0 ** -7 * s) + 1e-5


def to_np(t):
    import torch
    return t.detach().to(torch.float64).cpu().numpy()

"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
binding and the fp64 oracle on the same seeded inputs, and measure the error
the way the accuracy target is stated.

Error measure (per (batch, channel) row, normwise): for y,
    max_t |gpu - ref| / max_t |ref|
and for a state row max_n |gpu - ref| / max_n |ref|; the gate is the maximum
over rows.  Elementwise relative error is meaningless where y crosses zero.
Tolerances: 1e-4 for fp32 inputs, 2e-2 for bf16 inputs with fp32 state.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from selective_state_space_29_b200 import mamba_ssm as m
from selective_state_space_29_b200 import workloads as wl

TOL = {"f32": 1e-4, "bf16": 2e-2}


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def row_error(gpu: np.ndarray, ref: np.ndarray, axis: int) -> float:
    num = np.abs(gpu - ref).max(axis=axis)
    den = np.abs(ref).max(axis=axis)
    den = np.where(den > 0, den, 1.0)
    return float((num / den).max()) if num.size else 0.0


def gpu_scan(inp: dict, D=True, h0=None, chunk_len=0, general_a=False, method="zoh"):
    y, hf = m.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                             inp["D"] if D else None, initial_state=h0, chunk_len=chunk_len,
                             general_a=general_a, method=method)
    torch.cuda.synchronize()
    return y, hf


ORACLE_METHOD = {"zoh": 0, "euler": 1, "trapezoid": 2}


def oracle_scan_full(inp: dict, D=True, h0=None, method="zoh"):
    y, hf = oracle.scan(f64(inp["u"]), f64(inp["delta"]), f64(inp["A"]), f64(inp["B"]), f64(inp["C"]),
                        f64(inp["D"]) if D else None, h0=None if h0 is None else f64(h0),
                        method=ORACLE_METHOD[method])
    return y, hf


def sample_rows(batch: int, channels: int, count: int, seed: int = 0):
    """Deterministic (b, d) rows: the edges of the channel range and of the
    32-channel groups, plus random ones."""
    rng = np.random.default_rng(seed)
    picks = {(0, 0), (batch - 1, channels - 1), (0, min(31, channels - 1)), (batch - 1, min(32, channels - 1))}
    while len(picks) < min(count, batch * channels):
        picks.add((int(rng.integers(batch)), int(rng.integers(channels))))
    return sorted(picks)


def oracle_scan_rows(inp: dict, rows, D=True, h0=None):
    """Oracle y (len,) and final state (nstate,) for selected (b, d) rows,
    one oracle call per batch row over that row's selected channels."""
    out = {}
    by_b = {}
    for b, d in rows:
        by_b.setdefault(b, []).append(d)
    for b, ds in by_b.items():
        idx = torch.tensor(ds, device=inp["u"].device)
        u = f64(inp["u"][b:b + 1].index_select(2, idx))
        dl = f64(inp["delta"][b:b + 1].index_select(2, idx))
        A = f64(inp["A"].index_select(0, idx))
        Dv = f64(inp["D"].index_select(0, idx)) if D else None
        h = None if h0 is None else f64(h0[b:b + 1].index_select(1, idx))
        y, hf = oracle.scan(u, dl, A, f64(inp["B"][b:b + 1]), f64(inp["C"][b:b + 1]), Dv, h0=h)
        for i, d in enumerate(ds):
            out[(b, d)] = (y[0, :, i], hf[0, i])
    return out


def compare_rows(y_gpu: torch.Tensor, hf_gpu, ref: dict):
    ey = eh = 0.0
    for (b, d), (yr, hr) in ref.items():
        yg = f64(y_gpu[b, :, d])
        ey = max(ey, row_error(yg[None], yr[None], axis=1))
        if hf_gpu is not None:
            hg = f64(hf_gpu[b, d])
            eh = max(eh, row_error(hg[None], hr[None], axis=1))
    return ey, eh

"""GPU parity at the limits of the zero-order hold (page "Mamba SSM Nedir?
Transformer Alternatifi Rehberi (2026)", section "Ayrık Zamana Geçiş":
Abar = exp(Delta A), Bbar = (Delta A)^-1 (exp(Delta A) - 1) Delta B).

  Delta -> 0      Abar -> 1, Bbar -> 0: y = D x (the oracle is pinned there)
  Delta -> inf    Abar -> 0, Bbar -> -B/A: the memoryless map
                  y_t = sum_n C_t[n] (-B_t[n] / A_n) x_t + D x_t
  small |A|       slow decay, |Delta A| down to 1e-6: expm1 of tiny arguments
                  and long memory through the chunk and super-chunk hand-offs

Both kernel paths (A[d, n] = (n+1) A[d, 0], and A without that structure),
both dtypes, with and without the skip term, the scan and the single-token
state update; the same per-row error measure and tolerances as every other
parity test.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_29_b200 import workloads as wl
from selective_state_space_29_b200 import mamba_ssm as m
from tests.gpu_helpers import TOL, f64, gpu_scan, oracle_scan_full, row_error

pytestmark = pytest.mark.gpu
DEV = "cuda"

BASE = wl.ScanWorkload("limits", batch=2, length=1000, channels=200, nstate=16, dtype="bf16", seed=211)

DELTAS = {"tiny": (1e-14, 1e-14), "ten": (10.0, 10.0), "huge": (1e4, 1e4)}


def _run(w, chunk_len=0, D=True, method="zoh"):
    inp = wl.scan_inputs(w, DEV)
    y, hf = gpu_scan(inp, D=D, chunk_len=chunk_len, method=method)
    yr, hr = oracle_scan_full(inp, D=D, method=method)
    yg, hg = f64(y), f64(hf)
    assert np.isfinite(yg).all() and np.isfinite(hg).all()
    tol = TOL[w.dtype]
    ey, eh = row_error(yg, yr, axis=1), row_error(hg, hr, axis=2)
    assert ey <= tol, f"y error {ey:.3e} > {tol}"
    # with Delta -> 0 the final state is O(Delta): compare it absolutely there
    if w.delta_hi > 1e-10:
        assert eh <= tol, f"final state error {eh:.3e} > {tol}"
    else:
        assert np.abs(hg).max() <= 1e-9
    return inp, yg


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("a_mode", ["channel", "state"])
@pytest.mark.parametrize("which", sorted(DELTAS))
@pytest.mark.parametrize("chunk_len", [0, 128])
def test_scan_delta_limits(dtype, a_mode, which, chunk_len):
    lo, hi = DELTAS[which]
    w = BASE.with_(dtype=dtype, a_mode=a_mode, delta_lo=lo, delta_hi=hi)
    inp, yg = _run(w, chunk_len=chunk_len)
    if which == "tiny":
        # y = D x up to O(Delta) and the rounding of y to the I/O type
        dx = f64(inp["D"])[None, None, :] * f64(inp["u"])
        rel = 2.0 ** -8 if dtype == "bf16" else 1e-6
        assert np.abs(yg - dx).max() <= rel * np.abs(dx).max()
    _run(w, chunk_len=chunk_len, D=False)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("a_mode", ["small", "small_state"])
@pytest.mark.parametrize("chunk_len", [0, 128])
def test_scan_small_a(dtype, a_mode, chunk_len):
    w = BASE.with_(dtype=dtype, a_mode=a_mode)
    _run(w, chunk_len=chunk_len)
    _run(w, chunk_len=chunk_len, D=False)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("method", ["euler", "trapezoid"])
def test_scan_small_a_other_discretisations(dtype, method):
    _run(BASE.with_(dtype=dtype, a_mode="small_state"), D=False, method=method)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("a_mode", ["small", "channel"])
def test_scan_long_memory_across_super_chunks(dtype, a_mode):
    # two 32-channel groups: the sequence is cut into super-chunks, and with
    # small |A| and Delta down to 1e-4 the state entering each one matters
    w = wl.ScanWorkload("limits_long", batch=1, length=20000, channels=64, nstate=16, dtype=dtype,
                        delta_lo=1e-4, a_mode=a_mode, seed=212)
    _run(w, D=False)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("a_mode", ["channel", "random", "small", "small_state"])
@pytest.mark.parametrize("which", ["tiny", "huge", "normal"])
def test_state_update_limits(dtype, a_mode, which):
    lo, hi = DELTAS.get(which, (1e-3, 1e-1))
    w = wl.DecodeWorkload("limits", batch=3, channels=300, nstate=16, steps=20, dtype=dtype, delta_lo=lo,
                          delta_hi=hi, a_mode=a_mode, seed=213)
    prm = wl.decode_params(w, DEV)
    for D in (True, False):
        state = prm["state"].clone()
        ref = f64(prm["state"]).copy()
        ys, yrs = [], []
        for s in range(w.steps):
            st = wl.decode_step_inputs(w, s, DEV)
            y = m.state_update(state, st["x"], st["delta"], prm["A"], st["B"], st["C"], prm["D"] if D else None)
            yrs.append(oracle.state_update(ref, f64(st["x"]), f64(st["delta"]), f64(prm["A"]), f64(st["B"]),
                                           f64(st["C"]), f64(prm["D"]) if D else None))
            ys.append(f64(y))
        torch.cuda.synchronize()
        yg = np.stack(ys, axis=-1).reshape(-1, w.steps)
        yr = np.stack(yrs, axis=-1).reshape(-1, w.steps)
        tol = TOL[dtype]
        assert np.isfinite(yg).all()
        assert row_error(yg, yr, axis=1) <= tol
        assert row_error(f64(state).reshape(-1, w.nstate), ref.reshape(-1, w.nstate), axis=1) <= tol

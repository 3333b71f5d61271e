"""GPU parity of the scan's backward (mamba_selective_scan_backward) against the
fp64 oracle's reverse-mode gradients, through the C ABI: every gradient, both
dtypes, 4/8/16 states, initial state and final-state gradient, several tiles,
ragged channel groups, and sequences cut into super-chunks of one and of
several tiles (the last shape: 256 streams, 16 tiles)."""
import numpy as np
import pytest
import torch

import oracle as oracle_pkg
from selective_state_space_29_b200 import mamba_ssm as m
from selective_state_space_29_b200 import workloads as wl
from tests.gpu_helpers import TOL, f64, row_error

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _rows(name, a):
    """The gradient as rows over which the error is normalised, one row per
    (batch, channel) for du and dDelta (over tokens) and for the initial
    state's gradient (over states); one per channel for dA (over states);
    one per (batch, state) for dB and dC (over tokens); dD is one row."""
    a = np.asarray(a, dtype=np.float64)
    if name in ("du", "ddelta"):                 # (batch, len, channels)
        return a.transpose(0, 2, 1).reshape(-1, a.shape[1])
    if name in ("dB", "dC"):                     # (batch, len, nstate)
        return a.transpose(0, 2, 1).reshape(-1, a.shape[1])
    if name in ("dA", "d_initial_state", "dh0"):  # (channels, nstate) / (batch, channels, nstate)
        return a.reshape(-1, a.shape[-1])
    return a.reshape(1, -1)                      # dD


def _rel(name, g, r):
    return row_error(_rows(name, g), _rows(name, r), axis=1)


def _check(out, ref, D, tol):
    pairs = [("du", "du"), ("ddelta", "ddelta"), ("dA", "dA"), ("dB", "dB"), ("dC", "dC"),
             ("d_initial_state", "dh0")]
    if D is not None:
        pairs.append(("dD", "dD"))
    for mine, theirs in pairs:
        assert np.isfinite(f64(out[mine])).all(), mine
        e = _rel(mine, f64(out[mine]), ref[theirs])
        assert e <= tol, f"{mine}: per-row relative error {e:.2e} > {tol}"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 300, 100, 16), (1, 1000, 64, 8), (3, 200, 40, 4), (1, 64, 32, 16),
                                   (8, 1024, 1024, 16)])
@pytest.mark.parametrize("extras", [False, True])
def test_backward_matches_oracle(dtype, shape, extras):
    b, L, ch, n = shape
    w = wl.ScanWorkload("bwd", batch=b, length=L, channels=ch, nstate=n, dtype=dtype, a_mode="random",
                        seed=7 + L)
    inp = wl.scan_inputs(w, DEV)
    g = torch.Generator(device=DEV).manual_seed(3)
    dy = torch.randn(inp["u"].shape, generator=g, device=DEV).to(inp["u"].dtype)
    h0 = 0.5 * torch.randn((b, ch, n), generator=g, device=DEV) if extras else None
    dh = torch.randn((b, ch, n), generator=g, device=DEV) if extras else None
    D = inp["D"] if not extras else None
    out = m.selective_scan_backward(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D, dy,
                                    initial_state=h0, d_final_state=dh)
    torch.cuda.synchronize()
    ref = oracle_pkg.get().scan_backward(f64(inp["u"]), f64(inp["delta"]), f64(inp["A"]), f64(inp["B"]),
                                         f64(inp["C"]), None if D is None else f64(D), f64(dy),
                                         h0=None if h0 is None else f64(h0), dh_final=None if dh is None else f64(dh))
    _check(out, ref, D, TOL[dtype])


@pytest.mark.parametrize("length", [1, 3, 200])
@pytest.mark.parametrize("a_mode", ["small", "small_state"])
def test_backward_small_delta_a(length, a_mode):
    """fp32, |Delta A| from about 1e-7 to 1e-3 and h0 = 0: the part of dA that
    comes from d Bbar / dA (B x Delta^2 psi(Delta A)) is all of dA at one
    token and a large share at a few, so a cancellation in it shows."""
    w = wl.ScanWorkload("bwd_small", batch=2, length=length, channels=96, nstate=16, dtype="f32",
                        delta_lo=1e-4, delta_hi=1e-1, a_mode=a_mode, seed=41 + length)
    inp = wl.scan_inputs(w, DEV)
    g = torch.Generator(device=DEV).manual_seed(5)
    dy = torch.randn(inp["u"].shape, generator=g, device=DEV)
    out = m.selective_scan_backward(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], dy)
    torch.cuda.synchronize()
    ref = oracle_pkg.get().scan_backward(f64(inp["u"]), f64(inp["delta"]), f64(inp["A"]), f64(inp["B"]),
                                         f64(inp["C"]), f64(inp["D"]), f64(dy))
    _check(out, ref, inp["D"], TOL["f32"])


def test_backward_rejects_and_handles_edges():
    A = -torch.ones(8, 16, device=DEV)
    dA = torch.empty_like(A)
    lib = m.library()
    # 32 states: not built for the backward
    st = lib.mamba_selective_scan_backward(*([None] * 2), A.data_ptr(), *([None] * 3), None, None, None, None,
                                           None, dA.data_ptr(), dA.data_ptr(), dA.data_ptr(), None, None,
                                           1, 4, 8, 32, m.MAMBA_F32, None)
    assert st == m.MAMBA_ERR_UNSUPPORTED
    # len == 0: d_initial_state = d_final_state, sums zero
    dh = torch.randn(2, 8, 16, device=DEV)
    dh0 = torch.empty_like(dh)
    dB = torch.full((16,), 1.0, device=DEV)   # nothing is written to it at len 0
    st = lib.mamba_selective_scan_backward(None, None, A.data_ptr(), None, None, None, None, None, dh.data_ptr(),
                                           None, None, dA.data_ptr(), dB.data_ptr(), dB.data_ptr(), None,
                                           dh0.data_ptr(), 2, 0, 8, 16, m.MAMBA_F32, None)
    torch.cuda.synchronize()
    assert st == m.MAMBA_OK and torch.equal(dh0, dh) and (dA == 0).all()

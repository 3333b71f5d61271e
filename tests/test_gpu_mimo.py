"""GPU parity of the multi-input multi-output (MIMO) scan,
mamba_selective_scan_mimo, against the oracle's scan_mimo, through the C ABI.

Reading (the Mamba-3 page, "MIMO Mekanizmasının İşleyişi" and "Seçici Durum
Güncellemesindeki İyileştirmeler"): per channel, R inputs and R outputs share
one state and one step Delta; output r reads the state with its own C^(r).
Cases: both dtypes, R = 2 and 4, structured and general A, initial state,
no skip term, ragged channel groups and tiles, sequences long enough to be
cut into super-chunks, and the full-size bench shape on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_29_b200 import mamba_ssm as m
from selective_state_space_29_b200 import workloads as wl
from tests.gpu_helpers import TOL, f64, row_error

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check(w: wl.MimoWorkload, D=True, h0_std=None, general_a=False, rows=None):
    inp = wl.mimo_inputs(w, DEV)
    h0 = None
    if h0_std is not None:
        g = torch.Generator(device=DEV).manual_seed(9)
        h0 = h0_std * torch.randn((w.batch, w.channels, w.nstate), generator=g, device=DEV)
    y, hf = m.selective_scan_mimo(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"] if D else None,
                                  initial_state=h0, general_a=general_a)
    torch.cuda.synchronize()
    yg, hg = f64(y), f64(hf)
    assert np.isfinite(yg).all() and np.isfinite(hg).all()
    tol = TOL[w.dtype]
    if rows is None:
        yr, hr = oracle.scan_mimo(f64(inp["u"]), f64(inp["delta"]), f64(inp["A"]), f64(inp["B"]), f64(inp["C"]),
                                  f64(inp["D"]) if D else None, h0=None if h0 is None else f64(h0))
        # rows: one per (batch, output r, channel), over tokens
        ey = row_error(yg.transpose(0, 2, 3, 1).reshape(-1, w.length),
                       yr.transpose(0, 2, 3, 1).reshape(-1, w.length), axis=1)
        eh = row_error(hg, hr, axis=2)
    else:
        ey = eh = 0.0
        for b, d in rows:
            idx = torch.tensor([d], device=DEV)
            yr, hr = oracle.scan_mimo(f64(inp["u"][b:b + 1].index_select(3, idx)),
                                      f64(inp["delta"][b:b + 1].index_select(2, idx)),
                                      f64(inp["A"].index_select(0, idx)), f64(inp["B"][b:b + 1]),
                                      f64(inp["C"][b:b + 1]), f64(inp["D"].index_select(0, idx)) if D else None)
            ey = max(ey, row_error(yg[b, :, :, d].T, yr[0, :, :, 0].T, axis=1))
            eh = max(eh, row_error(hg[b, d][None], hr[0, 0][None], axis=1))
    assert ey <= tol, f"y error {ey:.3e} > {tol}"
    assert eh <= tol, f"final state error {eh:.3e} > {tol}"


SMALL = wl.MimoWorkload("mimo_small", batch=2, length=700, ranks=4, channels=200, nstate=16, dtype="bf16", seed=401)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("ranks", [2, 4])
@pytest.mark.parametrize("a_mode", ["channel", "random"])
def test_mimo_small(dtype, ranks, a_mode):
    _check(SMALL.with_(dtype=dtype, ranks=ranks, a_mode=a_mode))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_mimo_without_skip_and_with_initial_state(dtype):
    w = SMALL.with_(dtype=dtype, length=300)
    _check(w, D=False)
    _check(w, h0_std=0.5)
    _check(w, D=False, h0_std=0.5)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_mimo_general_flag_matches(dtype):
    _check(SMALL.with_(dtype=dtype, length=300), general_a=True)


@pytest.mark.parametrize("ranks", [2, 4])
@pytest.mark.parametrize("a_mode", ["channel", "small"])
def test_mimo_long_super_chunks(ranks, a_mode):
    # two channel groups: the sequence is cut into super-chunks joined by the correction kernel
    w = wl.MimoWorkload("mimo_long", batch=1, length=20000, ranks=ranks, channels=64, nstate=16, dtype="bf16",
                        delta_lo=1e-4, a_mode=a_mode, seed=402)
    _check(w, D=False, h0_std=0.3)


@pytest.mark.parametrize("shape", [(1, 1, 32), (3, 5, 33), (1, 17, 1), (2, 64, 96)])
def test_mimo_odd_shapes(shape):
    b, L, ch = shape
    _check(SMALL.with_(batch=b, length=L, channels=ch, dtype="f32"))


def test_mimo_bench_shape_sampled():
    w = wl.MIMO_WORKLOADS["mimo_mid_bf16"]
    rng = np.random.default_rng(5)
    rows = sorted({(0, 0), (w.batch - 1, w.channels - 1), (0, 31), (w.batch - 1, 32)} |
                  {(int(rng.integers(w.batch)), int(rng.integers(w.channels))) for _ in range(8)})
    _check(w, rows=rows)


def test_mimo_rejects_unsupported():
    x = torch.zeros(64, device=DEV)
    with pytest.raises(m.MambaError) as ei:
        m.mamba_selective_scan_mimo(x, x, x, x, x, None, None, x, None, 1, 1, 3, 4, 16, 0, m.MAMBA_F32)
    assert ei.value.status == m.MAMBA_ERR_UNSUPPORTED
    with pytest.raises(m.MambaError) as ei:
        m.mamba_selective_scan_mimo(x, x, x, x, x, None, None, x, None, 1, 1, 4, 4, 16, m.MAMBA_SCAN_EULER,
                                    m.MAMBA_F32)
    assert ei.value.status == m.MAMBA_ERR_UNSUPPORTED
    assert m.mamba_mimo_supported(4, 16) and not m.mamba_mimo_supported(4, 8)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("ranks", [2, 4])
@pytest.mark.parametrize("a_mode", ["channel", "random"])
def test_mimo_state_update_chain(dtype, ranks, a_mode):
    """20 single-token MIMO steps on 3 x 300 rows against the oracle's MIMO
    scan run one token at a time from the carried state."""
    w = wl.MimoWorkload("mimo_dec", batch=3, length=20, ranks=ranks, channels=300, nstate=16, dtype=dtype,
                        a_mode=a_mode, seed=403)
    inp = wl.mimo_inputs(w, DEV)
    g = torch.Generator(device=DEV).manual_seed(11)
    state = 0.1 * torch.randn((w.batch, w.channels, w.nstate), generator=g, device=DEV)
    ref = f64(state).copy()
    ys, yrs = [], []
    for t in range(w.length):
        y = m.state_update_mimo(state, inp["u"][:, t].contiguous(), inp["delta"][:, t].contiguous(), inp["A"],
                                inp["B"][:, t].contiguous(), inp["C"][:, t].contiguous(), inp["D"])
        yr, ref = oracle.scan_mimo(f64(inp["u"][:, t:t + 1]), f64(inp["delta"][:, t:t + 1]), f64(inp["A"]),
                                   f64(inp["B"][:, t:t + 1]), f64(inp["C"][:, t:t + 1]), f64(inp["D"]), h0=ref)
        ys.append(f64(y))
        yrs.append(yr[:, 0])
    torch.cuda.synchronize()
    yg = np.stack(ys, axis=-1).reshape(-1, w.length)
    yr = np.stack(yrs, axis=-1).reshape(-1, w.length)
    tol = TOL[dtype]
    assert row_error(yg, yr, axis=1) <= tol
    assert row_error(f64(state).reshape(-1, 16), ref.reshape(-1, 16), axis=1) <= tol


def test_mimo_state_update_chain_equals_scan():
    """L single-token MIMO steps from h0 = the MIMO scan from h0 over the same tokens."""
    w = wl.MimoWorkload("mimo_eq", batch=2, length=64, ranks=4, channels=96, nstate=16, dtype="f32", seed=404)
    inp = wl.mimo_inputs(w, DEV)
    h0 = 0.1 * torch.randn((w.batch, w.channels, 16), device=DEV)
    y_scan, hf = m.selective_scan_mimo(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                       initial_state=h0)
    state = h0.clone()
    ys = [m.state_update_mimo(state, inp["u"][:, t].contiguous(), inp["delta"][:, t].contiguous(), inp["A"],
                              inp["B"][:, t].contiguous(), inp["C"][:, t].contiguous(), inp["D"])
          for t in range(w.length)]
    torch.cuda.synchronize()
    yd = torch.stack(ys, dim=1)
    assert row_error(f64(yd).transpose(0, 2, 3, 1).reshape(-1, w.length),
                     f64(y_scan).transpose(0, 2, 3, 1).reshape(-1, w.length), axis=1) <= 1e-5
    assert row_error(f64(state), f64(hf), axis=2) <= 1e-5

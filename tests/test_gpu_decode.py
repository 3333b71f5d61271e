"""GPU parity of the recurrent state update (generation mode) against the
fp64 oracle's step chain, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_29_b200 import mamba_ssm as m
from selective_state_space_29_b200 import workloads as wl
from tests.gpu_helpers import TOL, f64, row_error

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _chain(w: wl.DecodeWorkload, rows=None, D=True):
    """Run w.steps updates on the GPU; follow the same steps in the oracle
    for all rows (rows=None) or for the selected (b, d) rows."""
    prm = wl.decode_params(w, DEV)
    state = prm["state"].clone()
    Dv = prm["D"] if D else None
    if rows is None:
        ref_state = f64(prm["state"]).copy()
        A = f64(prm["A"])
        Dr = f64(prm["D"]) if D else None
    else:
        bs = torch.tensor([b for b, _ in rows], device=DEV)
        ds = torch.tensor([d for _, d in rows], device=DEV)
        # each selected row becomes its own (batch 1, channel i) problem
        ref_state = f64(prm["state"][bs, ds]).reshape(len(rows), 1, w.nstate).copy()
        A_rows = f64(prm["A"][ds])
        D_rows = f64(prm["D"][ds]) if D else None
    ey = 0.0
    ys_gpu, ys_ref = [], []
    for s in range(w.steps):
        st = wl.decode_step_inputs(w, s, DEV)
        y = m.state_update(state, st["x"], st["delta"], prm["A"], st["B"], st["C"], Dv)
        if rows is None:
            yr = oracle.state_update(ref_state, f64(st["x"]), f64(st["delta"]), A, f64(st["B"]), f64(st["C"]), Dr)
            ys_gpu.append(f64(y))
            ys_ref.append(yr)
        else:
            yr = np.empty(len(rows))
            xs, dls = f64(st["x"][bs, ds]), f64(st["delta"][bs, ds])
            Bs, Cs = f64(st["B"][bs]), f64(st["C"][bs])
            for i in range(len(rows)):
                yr[i] = oracle.state_update(ref_state[i:i + 1], xs[i:i + 1].reshape(1, 1),
                                            dls[i:i + 1].reshape(1, 1), A_rows[i:i + 1], Bs[i:i + 1],
                                            Cs[i:i + 1], None if D_rows is None else D_rows[i:i + 1])[0, 0]
            ys_gpu.append(f64(y[bs, ds]))
            ys_ref.append(yr)
    torch.cuda.synchronize()
    yg = np.stack(ys_gpu, axis=-1)   # (..., steps)
    yrf = np.stack(ys_ref, axis=-1)
    if rows is None:
        ey = row_error(yg.reshape(-1, w.steps), yrf.reshape(-1, w.steps), axis=1)
        eh = row_error(f64(state).reshape(-1, w.nstate), ref_state.reshape(-1, w.nstate), axis=1)
    else:
        ey = row_error(yg, yrf, axis=1)
        sg = f64(state[bs, ds])
        eh = row_error(sg, ref_state.reshape(len(rows), w.nstate), axis=1)
    return ey, eh, state


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("a_mode", ["channel", "random"])
def test_decode_small_chain(dtype, a_mode):
    w = wl.DecodeWorkload("small", batch=3, channels=300, nstate=16, steps=50, dtype=dtype, a_mode=a_mode)
    ey, eh, _ = _chain(w)
    assert ey <= TOL[dtype] and eh <= TOL[dtype], (ey, eh)


@pytest.mark.parametrize("shape", [(1, 1), (1, 7), (5, 3), (2, 257)])
def test_decode_odd_shapes(shape):
    b, d = shape
    w = wl.DecodeWorkload("odd", batch=b, channels=d, nstate=16, steps=5, dtype="f32")
    ey, eh, _ = _chain(w)
    assert ey <= 1e-4 and eh <= 1e-4
    ey, eh, _ = _chain(w, D=False)
    assert ey <= 1e-4 and eh <= 1e-4


def test_decode_equals_scan():
    # L single-token updates from h0 = scan from h0 over the same L tokens
    w = wl.ScanWorkload("t", batch=2, length=64, channels=96, nstate=16, dtype="f32", seed=5)
    inp = wl.scan_inputs(w, DEV)
    h0 = 0.1 * torch.randn((w.batch, w.channels, 16), device=DEV)
    y_scan, hf = m.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                  initial_state=h0)
    state = h0.clone()
    ys = []
    for t in range(w.length):
        ys.append(m.state_update(state, inp["u"][:, t].contiguous(), inp["delta"][:, t].contiguous(), inp["A"],
                                 inp["B"][:, t].contiguous(), inp["C"][:, t].contiguous(), inp["D"]))
    torch.cuda.synchronize()
    yd = torch.stack(ys, dim=1)
    assert row_error(f64(yd), f64(y_scan), axis=1) <= 1e-5
    assert row_error(f64(state), f64(hf), axis=2) <= 1e-5


def test_decode_workload_sampled():
    """The 1000-step decode chain at full size (256 x 5120 x 16) on sampled rows."""
    w = wl.DECODE_WORKLOADS["decode_bf16"]
    rng = np.random.default_rng(4)
    rows = sorted({(0, 0), (255, 5119), (17, 31), (128, 32)} |
                  {(int(rng.integers(256)), int(rng.integers(5120))) for _ in range(28)})
    ey, eh, state = _chain(w, rows=rows)
    print(f"decode chain: y err {ey:.2e}, state err {eh:.2e} over {len(rows)} rows")
    assert ey <= TOL["bf16"] and eh <= TOL["bf16"]
    assert torch.isfinite(state).all()


@pytest.mark.parametrize("nstate", [4, 8, 32])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_other_state_counts(nstate, dtype):
    # nstate/4 lanes per (batch, channel) row: 1, 2 and 8 lanes
    w = wl.DecodeWorkload("n", batch=5, channels=300, nstate=nstate, steps=20, dtype=dtype, a_mode="random")
    ey, eh, _ = _chain(w)
    assert ey <= TOL[dtype] and eh <= TOL[dtype], (ey, eh)

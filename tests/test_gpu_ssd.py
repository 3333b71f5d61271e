"""GPU parity of Mamba-2's scalar-A scan (`mamba_ssd_scan`, the chunked
tensor-core form) against the fp64 oracle's recurrence, through the C ABI.

Small cases are compared over whole outputs: ragged last chunks, lengths
below one chunk, one and several super-chunks (forced and automatic), 16,
32 and 64 states, exponential Euler, an initial state, no skip term.  The
full-size workloads are compared on sampled heads (every channel of each),
in the launch configuration the benchmark uses.  Tolerance: the bf16 one of
the scan (2e-2, per (batch, channel) row, normwise).
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
P = 64


def _h0(w, std=0.3, seed=7):
    g = torch.Generator(device=DEV).manual_seed(seed)
    return std * torch.randn((w.batch, w.channels, w.nstate), generator=g, device=DEV)


def _oracle(inp, heads=None, D=True, h0=None, method="zoh"):
    """Oracle y, final state for all heads or the listed ones."""
    x, dt, A, Dv = inp["x"], inp["dt"], inp["A"], inp["D"]
    if heads is not None:
        idx = torch.tensor(heads, device=x.device)
        ch = (idx[:, None] * P + torch.arange(P, device=x.device)[None, :]).reshape(-1)
        x = x.index_select(2, ch)
        dt = dt.index_select(2, idx)
        A = A.index_select(0, idx)
        Dv = Dv.index_select(0, ch)
        if h0 is not None:
            h0 = h0.index_select(1, ch)
    return oracle.ssd_scan(f64(x), f64(dt), f64(A), f64(inp["B"]), f64(inp["C"]), f64(Dv) if D else None,
                           h0=None if h0 is None else f64(h0), headdim=P,
                           method={"zoh": 0, "euler": 1}[method])


def _check(w, supers=0, D=True, h0=None, method="zoh", seed=None, heads=None, normwise="row"):
    """normwise="row": the scan's measure, per (batch, channel) row over
    time.  normwise="all": over the whole output, for rows shorter than a
    chunk -- there max_t |y| is one or a few tokens' |y|, which cancellation
    between C.h and D x can make arbitrarily small, while the matrix form's
    bf16 operands carry errors relative to each term, not to their sum."""
    inp = wl.ssd_inputs(w, DEV, seed)
    y, hf = m.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"] if D else None,
                       initial_state=h0, supers=supers, method=method)
    torch.cuda.synchronize()
    yr, hr = _oracle(inp, heads, D, h0, method)
    if heads is not None:
        ch = torch.tensor(np.concatenate([np.arange(h * P, (h + 1) * P) for h in heads]), device=y.device)
        y, hf = y.index_select(2, ch), hf.index_select(1, ch)
    yg, hg = f64(y), f64(hf)
    assert np.isfinite(yg).all() and np.isfinite(hg).all()
    if normwise == "all":
        ey = float(np.abs(yg - yr).max() / np.abs(yr).max()) if w.length else 0.0
    else:
        ey = row_error(yg, yr, axis=1) if w.length else 0.0
    eh = row_error(hg, hr, axis=2)
    tol = TOL["bf16"]
    assert ey <= tol, f"y error {ey:.3e} > {tol}"
    assert eh <= tol, f"final state error {eh:.3e} > {tol}"
    return ey, eh


SMALL = wl.SsdWorkload("ssd_small", batch=2, length=1000, heads=3, headdim=P, nstate=16, seed=201)


@pytest.mark.parametrize("supers", [0, 1, 3, 16])
def test_ssd_small_super_splits(supers):
    # 1000 tokens = 15 full chunks + 40; 0 = automatic (many super-chunks here)
    _check(SMALL, supers=supers)


@pytest.mark.parametrize("nstate", [16, 32, 64])
@pytest.mark.parametrize("supers", [0, 1])
def test_ssd_state_counts(nstate, supers):
    _check(SMALL.with_(nstate=nstate, length=700), supers=supers)


@pytest.mark.parametrize("supers", [0, 1])
def test_ssd_euler(supers):
    _check(SMALL, supers=supers, method="euler")


@pytest.mark.parametrize("supers", [0, 1, 4])
def test_ssd_initial_state(supers):
    w = SMALL.with_(length=900)
    _check(w, supers=supers, h0=_h0(w))


def test_ssd_no_skip_term():
    # without D x the outputs are the state-space part alone
    _check(SMALL, supers=1, D=False)
    _check(SMALL, supers=0, D=False)


@pytest.mark.parametrize("length", [1, 17, 63, 64, 65, 128, 129])
def test_ssd_short_and_ragged_lengths(length):
    w = SMALL.with_(length=length, batch=3, heads=2)
    nw = "all" if length < 64 else "row"
    _check(w, supers=1, h0=_h0(w), normwise=nw)
    _check(w, supers=0, normwise=nw)


def test_ssd_wide_delta_range():
    # steps up to 1: decays over a chunk reach exp(-1000), far below fp32's range
    _check(SMALL.with_(delta_lo=1e-4, delta_hi=1.0), supers=0)


def test_ssd_len_zero_copies_initial_state():
    w = SMALL.with_(length=0)
    inp = wl.ssd_inputs(w, DEV)
    h0 = _h0(w)
    _, hf = m.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], initial_state=h0)
    torch.cuda.synchronize()
    assert torch.equal(hf, h0)
    _, hf = m.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"])
    torch.cuda.synchronize()
    assert torch.count_nonzero(hf) == 0


def test_ssd_deterministic():
    inp = wl.ssd_inputs(SMALL, DEV)
    outs = [m.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"]) for _ in range(2)]
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_ssd_matches_selective_scan_path():
    """The same problem through the selective scan (A and delta broadcast to
    channels): the two CUDA paths agree within the bf16 tolerance."""
    w = SMALL.with_(length=800)
    inp = wl.ssd_inputs(w, DEV)
    y1, h1 = m.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"])
    head = torch.arange(w.channels, device=DEV) // P
    delta = inp["dt"].index_select(2, head).contiguous()
    A = inp["A"][head][:, None].expand(w.channels, w.nstate).contiguous()
    y2, h2 = m.selective_scan(inp["x"], delta, A, inp["B"], inp["C"], inp["D"], general_a=True)
    torch.cuda.synchronize()
    assert row_error(f64(y1), f64(y2), axis=1) <= 2 * TOL["bf16"]
    assert row_error(f64(h1), f64(h2), axis=2) <= 2 * TOL["bf16"]


def test_ssd_mid_workload_sampled_heads():
    w = wl.SSD_WORKLOADS["ssd_mid_bf16"]
    _check(w, heads=[0, 17, w.heads - 1])


@pytest.mark.slow
def test_ssd_long_workload_sampled_head():
    w = wl.SSD_WORKLOADS["ssd_long_bf16"]
    _check(w, heads=[w.heads - 1])


def test_ssd_graph_capture_replays_the_eager_result():
    # the small shape uses several super-chunks, so the captured call also
    # allocates and frees its aggregate scratch inside the graph
    inp = wl.ssd_inputs(SMALL, DEV)
    args = (inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"])
    y0, h0 = m.ssd_scan(*args)
    y, hf = torch.empty_like(y0), torch.empty_like(h0)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        m.ssd_scan(*args, y=y, final_state=hf)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, y0) and torch.equal(hf, h0)

"""GPU parity of the selective scan against the fp64 oracle, through the C ABI.

Small cases are compared element by element over whole outputs (several
32-channel groups, a ragged last group, ragged time tiles, forced chunk
splits); the full-size workloads are compared on sampled (batch, channel)
rows, which the oracle computes one by one, in the same launch configuration
the benchmark uses.
"""
import numpy as np
import pytest
import torch

from selective_state_space_29_b200 import mamba_ssm as m
from selective_state_space_29_b200 import workloads as wl
from tests.gpu_helpers import (TOL, compare_rows, f64, gpu_scan, oracle_scan_full, oracle_scan_rows,
                               row_error, sample_rows)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check_full(w: wl.ScanWorkload, chunk_len=0, general_a=False, D=True, h0_std=None, seed=None, method="zoh"):
    inp = wl.scan_inputs(w, DEV, seed)
    h0 = None
    if h0_std is not None:
        g = torch.Generator(device=DEV).manual_seed(7)
        h0 = h0_std * torch.randn((w.batch, w.channels, w.nstate), generator=g, device=DEV)
    y, hf = gpu_scan(inp, D=D, h0=h0, chunk_len=chunk_len, general_a=general_a, method=method)
    yr, hr = oracle_scan_full(inp, D=D, h0=h0, method=method)
    ey = row_error(f64(y), yr, axis=1)
    eh = row_error(f64(hf), hr, axis=2)
    tol = TOL[w.dtype]
    assert np.isfinite(f64(y)).all() and np.isfinite(f64(hf)).all()
    assert ey <= tol, f"y error {ey:.3e} > {tol}"
    assert eh <= tol, f"final state error {eh:.3e} > {tol}"
    return ey, eh


SMALL = wl.ScanWorkload("small", batch=2, length=1000, channels=200, nstate=16, dtype="bf16", seed=101)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("a_mode", ["s4d", "channel", "state", "random"])
def test_scan_small_all_paths(dtype, a_mode):
    _check_full(SMALL.with_(dtype=dtype, a_mode=a_mode))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_scan_plain_load_path(dtype):
    # 100 channels: a row is 200 (bf16) / 400 (fp32) bytes; bf16 rows are not a
    # multiple of 16 bytes, so the tile loads cannot use TMA there
    _check_full(SMALL.with_(channels=100, dtype=dtype, length=300))


@pytest.mark.parametrize("chunk_len", [1, 37, 128, 999, 1000, 5000])
def test_scan_forced_chunks(chunk_len):
    # the associative chunk combine on any split, including one token per chunk
    _check_full(SMALL.with_(length=600 if chunk_len == 1 else 1000), chunk_len=chunk_len)


@pytest.mark.parametrize("chunk_len", [0, 64])
def test_scan_general_flag_matches(chunk_len):
    _check_full(SMALL.with_(a_mode="channel"), chunk_len=chunk_len, general_a=True)


@pytest.mark.parametrize("chunk_len", [0, 100])
def test_scan_initial_state(chunk_len):
    _check_full(SMALL.with_(dtype="f32", length=400), chunk_len=chunk_len, h0_std=0.5)
    _check_full(SMALL.with_(length=400), chunk_len=chunk_len, h0_std=0.5)


def test_scan_without_skip_term():
    # D = None: y is the pure state path, so state errors cannot hide under D x
    _check_full(SMALL.with_(dtype="f32"), D=False)
    _check_full(SMALL, D=False)


@pytest.mark.parametrize("shape", [(1, 1, 32), (3, 7, 33), (1, 33, 1), (5, 64, 64), (1, 4096, 31)])
def test_scan_odd_shapes(shape):
    b, L, Dc = shape
    _check_full(SMALL.with_(batch=b, length=L, channels=Dc, dtype="f32"))
    _check_full(SMALL.with_(batch=b, length=L, channels=Dc))


def test_scan_long_few_channels_autochunk():
    # 2 groups only: the planner splits the sequence into super-chunks
    _check_full(SMALL.with_(batch=1, length=20000, channels=64, delta_lo=1e-4), D=False)


def test_scan_len_zero_and_empty():
    w = SMALL.with_(length=0)
    inp = wl.scan_inputs(w, DEV)
    hf = torch.full((w.batch, w.channels, w.nstate), 7.0, device=DEV)
    m.mamba_selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["u"], hf,
                           w.batch, 0, w.channels, 16, m.MAMBA_BF16)
    torch.cuda.synchronize()
    assert (hf == 0).all()
    h0 = torch.randn_like(hf)
    m.mamba_selective_scan_ex(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], h0, inp["u"],
                              hf, w.batch, 0, w.channels, 16, 0, 0, m.MAMBA_BF16)
    torch.cuda.synchronize()
    assert torch.equal(hf, h0)
    # batch 0 / channels 0: no-op
    m.mamba_selective_scan(None, None, None, None, None, None, None, None, 0, 10, 10, 16, m.MAMBA_BF16)
    m.mamba_selective_scan(None, None, None, None, None, None, None, None, 2, 10, 0, 16, m.MAMBA_BF16)


def test_scan_state_layout_by_index():
    # one channel gets an impulse, every other input is zero: only the state
    # entries [b, d, :] of that row may become non-zero, and they must match
    w = SMALL.with_(batch=2, length=8, channels=40, dtype="f32")
    inp = wl.scan_inputs(w, DEV)
    inp["u"].zero_()
    inp["u"][1, 3, 37] = 1.0
    y, hf = gpu_scan(inp)
    nz = torch.nonzero(hf.abs().sum(dim=2))
    assert nz.tolist() == [[1, 37]]
    _, hr = oracle_scan_full(inp)
    assert row_error(f64(hf[1, 37])[None], hr[1, 37][None], axis=1) <= 1e-5


def test_scan_deterministic():
    inp = wl.scan_inputs(SMALL, DEV)
    y1, h1 = gpu_scan(inp)
    y2, h2 = gpu_scan(inp)
    assert torch.equal(y1, y2) and torch.equal(h1, h2)


def test_scan_output_does_not_write_outside():
    # canary bands around y and the final state
    w = SMALL.with_(channels=72, length=333)
    inp = wl.scan_inputs(w, DEV)
    pad = 4096
    ybuf = torch.full((pad + w.batch * w.length * w.channels + pad,), float("nan"), device=DEV,
                      dtype=torch.bfloat16)
    hbuf = torch.full((pad + w.batch * w.channels * 16 + pad,), float("nan"), device=DEV)
    y = ybuf[pad:pad + w.batch * w.length * w.channels].view(w.batch, w.length, w.channels)
    hf = hbuf[pad:pad + w.batch * w.channels * 16].view(w.batch, w.channels, 16)
    m.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], y=y, final_state=hf)
    torch.cuda.synchronize()
    assert torch.isnan(ybuf[:pad].float()).all() and torch.isnan(ybuf[-pad:].float()).all()
    assert torch.isnan(hbuf[:pad]).all() and torch.isnan(hbuf[-pad:]).all()
    assert torch.isfinite(y.float()).all() and torch.isfinite(hf).all()


# --- full-size workloads on sampled rows ---------------------------------------

@pytest.mark.parametrize("name", ["tiny_f32"])
def test_workload_tiny_full(name):
    ey, eh = _check_full(wl.SCAN_WORKLOADS[name])
    print(f"{name}: y err {ey:.2e}, state err {eh:.2e}")


@pytest.mark.parametrize("name,count", [("mid_bf16", 24), ("large_bf16", 24), ("long_bf16", 12)])
def test_workload_sampled(name, count):
    w = wl.SCAN_WORKLOADS[name]
    inp = wl.scan_inputs(w, DEV)
    y, hf = gpu_scan(inp)
    rows = sample_rows(w.batch, w.channels, count, seed=3)
    ref = oracle_scan_rows(inp, rows)
    ey, eh = compare_rows(y, hf, ref)
    print(f"{name}: y err {ey:.2e}, state err {eh:.2e} over {len(rows)} rows")
    assert ey <= TOL[w.dtype] and eh <= TOL[w.dtype]
    # properties that hold at any size: finite everywhere, state shape
    assert torch.isfinite(hf).all()
    assert hf.shape == (w.batch, w.channels, w.nstate)
    del inp, y, hf
    torch.cuda.empty_cache()


@pytest.mark.parametrize("a_mode", ["channel", "random"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_scan_more_groups_than_warps(a_mode, dtype):
    # 40 x 32 groups of 32 channels: more streams than resident consumer warps,
    # so every warp runs several groups, without super-chunks
    w = SMALL.with_(batch=40, length=96, channels=1024, a_mode=a_mode, dtype=dtype)
    plan = m.mamba_scan_plan(w.batch, w.length, w.channels, 16, 0, m.dtype_code(w.torch_dtype))
    assert plan.supers == 1
    _check_full(w)


# --- exponential-Euler and trapezoidal discretisations (flags of mamba_selective_scan_ex) ---

@pytest.mark.parametrize("method", ["euler", "trapezoid"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("a_mode", ["s4d", "random"])
def test_scan_methods_small(method, dtype, a_mode):
    _check_full(SMALL.with_(dtype=dtype, a_mode=a_mode), method=method)


@pytest.mark.parametrize("chunk_len", [1, 37, 999])
def test_scan_trapezoid_across_chunks(chunk_len):
    # the previous token's input term crosses every chunk and super-chunk border
    _check_full(SMALL.with_(length=600 if chunk_len == 1 else 1000), chunk_len=chunk_len, method="trapezoid")


@pytest.mark.parametrize("method", ["euler", "trapezoid"])
def test_scan_methods_initial_state_and_super_chunks(method):
    _check_full(SMALL.with_(dtype="f32", length=400), chunk_len=100, h0_std=0.5, method=method)
    _check_full(SMALL.with_(batch=1, length=20000, channels=64, delta_lo=1e-4), D=False, method=method)


def test_scan_methods_flags_rejected_together():
    inp = wl.scan_inputs(SMALL, DEV)
    y = torch.empty_like(inp["u"])
    st = m.library().mamba_selective_scan_ex(
        inp["u"].data_ptr(), inp["delta"].data_ptr(), inp["A"].data_ptr(), inp["B"].data_ptr(),
        inp["C"].data_ptr(), inp["D"].data_ptr(), None, y.data_ptr(), None, SMALL.batch, SMALL.length,
        SMALL.channels, 16, 0, m.MAMBA_SCAN_EULER | m.MAMBA_SCAN_TRAPEZOID, m.MAMBA_BF16, None)
    assert st == m.MAMBA_ERR_INVALID_ARG


# --- other state counts -------------------------------------------------------------------

@pytest.mark.parametrize("nstate", [4, 8, 32])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("a_mode", ["s4d", "random"])
def test_scan_other_state_counts(nstate, dtype, a_mode):
    _check_full(SMALL.with_(nstate=nstate, dtype=dtype, a_mode=a_mode))


@pytest.mark.parametrize("nstate", [4, 32])
def test_scan_other_state_counts_chunked_and_initial_state(nstate):
    _check_full(SMALL.with_(nstate=nstate, length=700), chunk_len=100, h0_std=0.5)
    _check_full(SMALL.with_(nstate=nstate, batch=1, length=20000, channels=64, delta_lo=1e-4), D=False)


@pytest.mark.parametrize("nstate", [8, 32])
def test_scan_other_state_counts_methods(nstate):
    _check_full(SMALL.with_(nstate=nstate, length=500), method="trapezoid", chunk_len=123)
    _check_full(SMALL.with_(nstate=nstate, length=500, dtype="f32"), method="euler")


@pytest.mark.parametrize("shape", ["groups", "super_chunks"])
def test_scan_capture_in_cuda_graph(shape):
    # the call only enqueues stream work (stream-ordered scratch, kernels), so
    # it can be captured once and replayed; replays equal the eager call bit for bit
    w = SMALL if shape == "groups" else SMALL.with_(batch=1, length=20000, channels=64)
    inp = wl.scan_inputs(w, DEV)
    y0, h0 = gpu_scan(inp)
    y = torch.empty_like(y0)
    hf = torch.empty_like(h0)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        m.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], y=y, final_state=hf)
    for _ in range(2):
        y.zero_()
        hf.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, y0) and torch.equal(hf, h0)
    del g

"""mamba_selective_scan_host: the scan on host buffers, copies pipelined with
the scan piece by piece, checked against the fp64 oracle (whole outputs on a
small case with several pieces and a ragged last piece; sampled rows on the
mid workload, as the benchmark's end-to-end leg runs it)."""
import numpy as np
import pytest
import torch

from selective_state_space_29_b200 import mamba_ssm as m
from selective_state_space_29_b200 import workloads as wl
from tests.gpu_helpers import TOL, compare_rows, f64, oracle_scan_full, oracle_scan_rows, row_error, sample_rows

pytestmark = pytest.mark.gpu


def _host(inp):
    return {k: v.cpu().pin_memory() for k, v in inp.items()}


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("piece_len", [0, 256, 300, 5000])
def test_host_scan_small(dtype, piece_len):
    w = wl.ScanWorkload("small", batch=2, length=1000, channels=200, nstate=16, dtype=dtype, seed=101)
    inp = wl.scan_inputs(w, "cuda")
    h = _host(inp)
    y, hf = m.selective_scan_host(h["u"], h["delta"], h["A"], h["B"], h["C"], h["D"], piece_len=piece_len)
    yr, hr = oracle_scan_full(inp)
    assert row_error(f64(y), yr, axis=1) <= TOL[dtype]
    assert row_error(f64(hf), hr, axis=2) <= TOL[dtype]


def test_host_scan_without_skip_and_state():
    w = wl.ScanWorkload("small", batch=3, length=777, channels=64, nstate=16, dtype="bf16", seed=5)
    inp = wl.scan_inputs(w, "cuda")
    h = _host(inp)
    y = torch.empty(h["u"].shape, dtype=h["u"].dtype).pin_memory()
    m.mamba_selective_scan_host(h["u"], h["delta"], h["A"], h["B"], h["C"], None, y, None, w.batch, w.length,
                                w.channels, 16, 128, m.MAMBA_BF16)
    torch.cuda.synchronize()
    yr, _ = oracle_scan_full(inp, D=False)
    assert row_error(f64(y), yr, axis=1) <= TOL["bf16"]


def test_host_scan_mid_sampled():
    w = wl.SCAN_WORKLOADS["mid_bf16"]
    inp = wl.scan_inputs(w, "cuda")
    h = _host(inp)
    y, hf = m.selective_scan_host(h["u"], h["delta"], h["A"], h["B"], h["C"], h["D"])
    rows = sample_rows(w.batch, w.channels, 12, seed=9)
    ref = oracle_scan_rows(inp, rows)
    ey, eh = compare_rows(y.cuda(), hf.cuda(), ref)
    assert ey <= TOL["bf16"] and eh <= TOL["bf16"]
    assert torch.isfinite(hf).all()


def test_host_scan_len_zero_and_errors():
    fs = torch.full((2, 8, 16), 3.0)
    A = -torch.ones(8, 16)
    st = m.library().mamba_selective_scan_host(None, None, A.data_ptr(), None, None, None, None, fs.data_ptr(),
                                               2, 0, 8, 16, 0, m.MAMBA_F32, None)
    assert st == m.MAMBA_OK and (fs == 0).all()
    st = m.library().mamba_selective_scan_host(None, None, A.data_ptr(), None, None, None, None, None,
                                               2, 10, 8, 16, 0, m.MAMBA_F32, None)
    assert st == m.MAMBA_ERR_INVALID_ARG

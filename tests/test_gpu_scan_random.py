"""Randomised GPU parity: 48 seeded configurations drawn over every option of
mamba_selective_scan_ex at once (batch, length, channel count with ragged
groups, state count, dtype, A structure, forced chunking, skip term, initial
state, discretisation), each compared element by element with the fp64
oracle.  The draws are fixed by the case index, so a failure reproduces."""
import numpy as np
import pytest
import torch

from selective_state_space_29_b200 import workloads as wl
from tests.gpu_helpers import TOL, f64, gpu_scan, oracle_scan_full, row_error

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(i: int):
    r = np.random.default_rng(1000 + i)
    w = wl.ScanWorkload(
        f"rand{i}", batch=int(r.integers(1, 5)), length=int(r.integers(1, 700)),
        channels=int(r.choice([1, 7, 31, 32, 33, 64, 100, 200, 300])),
        nstate=int(r.choice([4, 8, 16, 32])), dtype=str(r.choice(["bf16", "f32"])),
        delta_lo=float(r.choice([1e-4, 1e-3])), a_mode=str(r.choice(["s4d", "channel", "state", "random"])),
        seed=int(r.integers(1, 1 << 30)))
    chunk = int(r.choice([0, 0, 1, 17, 64, 100, 333]))
    if chunk == 1:
        w = w.with_(length=min(w.length, 200))
    method = str(r.choice(["zoh", "zoh", "euler", "trapezoid"]))
    return w, chunk, method, bool(r.integers(0, 2)), bool(r.integers(0, 2))


@pytest.mark.parametrize("i", range(48))
def test_random_configuration(i):
    w, chunk, method, use_d, use_h0 = _case(i)
    inp = wl.scan_inputs(w, DEV)
    h0 = None
    if use_h0:
        g = torch.Generator(device=DEV).manual_seed(i)
        h0 = 0.3 * torch.randn((w.batch, w.channels, w.nstate), generator=g, device=DEV)
    y, hf = gpu_scan(inp, D=use_d, h0=h0, chunk_len=chunk, method=method)
    yr, hr = oracle_scan_full(inp, D=use_d, h0=h0, method=method)
    tol = TOL[w.dtype]
    desc = f"{w} chunk={chunk} method={method} D={use_d} h0={use_h0}"
    assert np.isfinite(f64(y)).all() and np.isfinite(f64(hf)).all(), desc
    assert row_error(f64(y), yr, axis=1) <= tol, desc
    assert row_error(f64(hf), hr, axis=2) <= tol, desc

"""mamba_selective_scan_noalloc: the scan for callers that may not allocate
device memory inside an operation (inference runtimes and plugin hosts that
plan all device memory ahead, fixed memory budgets, processes whose memory
belongs to another allocator).  Its scratch is a fixed device array inside
the library.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it must also pass on its own in a
fresh process (the first call on the device sets up the array's address).
"""
import pytest
import torch

from selective_state_space_29_b200 import mamba_ssm as m
from selective_state_space_29_b200 import workloads as wl
from tests.gpu_helpers import TOL, compare_rows, oracle_scan_rows, sample_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _scan_both(inp, w):
    """The allocating entry point and the no-alloc one on the same inputs."""
    y_ref = torch.empty_like(inp["u"])
    h_ref = torch.empty((w.batch, w.channels, w.nstate), device=DEV)
    m.mamba_selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], y_ref, h_ref,
                           w.batch, w.length, w.channels, w.nstate, m.dtype_code(w.torch_dtype))
    y = torch.full_like(inp["u"], float("nan"))
    h = torch.full((w.batch, w.channels, w.nstate), float("nan"), device=DEV)
    m.mamba_selective_scan_noalloc(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], y, h,
                                   w.batch, w.length, w.channels, w.nstate, m.dtype_code(w.torch_dtype))
    torch.cuda.synchronize()
    return y, h, y_ref, h_ref


@pytest.mark.parametrize("w", [
    wl.ScanWorkload("na_small", 2, 1000, 200, 16, "bf16", seed=71),
    wl.ScanWorkload("na_f32", 1, 300, 96, 16, "f32", seed=72),
    wl.ScanWorkload("na_long", 1, 20000, 64, 16, "bf16", delta_lo=1e-4, seed=73),   # split into super-chunks
    wl.SCAN_WORKLOADS["mid_bf16"],
], ids=lambda w: w.name)
def test_noalloc_matches_allocating_scan_twice(w):
    tol = TOL[w.dtype]
    for call in range(2):   # two calls in a row, different inputs: nothing stale may leak through
        inp = wl.scan_inputs(w, DEV, seed=w.seed + 17 * call)
        y, h, y_ref, h_ref = _scan_both(inp, w)
        assert torch.isfinite(y.float()).all() and torch.isfinite(h).all()
        # the same kernels on the same split, only the scratch differs: bit for bit
        assert torch.equal(y, y_ref) and torch.equal(h, h_ref)
        # and a few rows against the fp64 oracle
        rows = sample_rows(w.batch, w.channels, 6, seed=call)
        ey, eh = compare_rows(y, h, oracle_scan_rows(inp, rows))
        assert ey <= tol and eh <= tol, (ey, eh)
    assert m.mamba_get_device_error(clear=False) == m.MAMBA_OK


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 1 x 1,048,576 x 2048 needs about 70 MB of scratch, more than the 16 MiB array
    plan = m.mamba_scan_plan(1, 1 << 20, 2048, 16, 0, m.MAMBA_BF16)
    assert plan.scratch_bytes > 16 << 20
    x = torch.zeros(16, device=DEV, dtype=torch.bfloat16)   # never read: rejected on the host
    with pytest.raises(m.MambaError) as ei:
        m.mamba_selective_scan_noalloc(x, x, x, x, x, None, x, None, 1, 1 << 20, 2048, 16, m.MAMBA_BF16)
    assert ei.value.status == m.MAMBA_ERR_UNSUPPORTED


def test_noalloc_does_not_take_device_memory():
    """The library counts every scratch allocation it makes in this process:
    the allocating scan adds one per call, the no-alloc scan none.  (Free
    device memory is no measure on a GPU other processes share.)"""
    w = wl.ScanWorkload("na_mem", 2, 512, 128, 16, "bf16", seed=74)
    inp = wl.scan_inputs(w, DEV)
    y = torch.empty_like(inp["u"])
    h = torch.empty((w.batch, w.channels, w.nstate), device=DEV)
    args = (inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], y, h,
            w.batch, w.length, w.channels, w.nstate, m.MAMBA_BF16)
    before = m.mamba_debug_scratch_allocations()
    for _ in range(3):
        m.mamba_selective_scan_noalloc(*args)
    torch.cuda.synchronize()
    assert m.mamba_debug_scratch_allocations() == before
    m.mamba_selective_scan(*args)
    torch.cuda.synchronize()
    assert m.mamba_debug_scratch_allocations() == before + 1

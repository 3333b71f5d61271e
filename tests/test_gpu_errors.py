"""Error behaviour of the C ABI on a GPU: argument errors, and a bounded
device wait that runs out without faulting (the context stays usable)."""
import pytest
import torch

from selective_state_space_29_b200 import mamba_ssm as m
from selective_state_space_29_b200 import workloads as wl
from tests.gpu_helpers import gpu_scan

pytestmark = pytest.mark.gpu


def test_argument_errors_raise():
    w = wl.ScanWorkload("e", 1, 16, 32, 16, "bf16")
    inp = wl.scan_inputs(w, "cuda")
    with pytest.raises(m.MambaError) as ei:
        m.mamba_selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], None, None, None,
                               1, 16, 32, 16, m.MAMBA_BF16)
    assert ei.value.status == m.MAMBA_ERR_INVALID_ARG
    with pytest.raises(m.MambaError) as ei:
        m.mamba_selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], None, inp["u"], None,
                               1, 16, 32, 12, m.MAMBA_BF16)
    assert ei.value.status == m.MAMBA_ERR_UNSUPPORTED


def test_bounded_wait_expires_and_context_survives():
    assert m.mamba_get_device_error(clear=True) == m.MAMBA_OK
    m.mamba_debug_expire_wait(2_000_000)          # 2 ms limit on a barrier nobody completes
    assert m.mamba_get_device_error(clear=False) == m.MAMBA_ERR_TIMEOUT
    assert m.mamba_get_device_error(clear=True) == m.MAMBA_ERR_TIMEOUT
    assert m.mamba_get_device_error(clear=False) == m.MAMBA_OK
    # the context still works: a scan runs and is finite
    inp = wl.scan_inputs(wl.ScanWorkload("e", 1, 64, 64, 16, "bf16"), "cuda")
    y, hf = gpu_scan(inp)
    assert torch.isfinite(y.float()).all()
    assert m.mamba_get_device_error(clear=False) == m.MAMBA_OK


def test_scan_leaves_no_device_error():
    inp = wl.scan_inputs(wl.ScanWorkload("e", 1, 5000, 64, 16, "bf16"), "cuda")
    m.mamba_get_device_error(clear=True)
    gpu_scan(inp, chunk_len=50)
    gpu_scan(inp)
    assert m.mamba_get_device_error(clear=False) == m.MAMBA_OK

"""Host-side checks of the C ABI (no GPU needed, no compute calls).

The library is built in-tree for sm_100a (nvcc cross-compiles without a GPU),
loaded with ctypes, and every entry point that include/mamba_ssm.h declares
must be exported.  Only calls that return before touching the device are
made here: status strings, the supported-nstate query, and argument checks
that reject or short-circuit a call on the host.
"""
import ctypes
import os
import re

import pytest

from selective_state_space_29_b200 import build as lib_build
from selective_state_space_29_b200 import mamba_ssm as m

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mamba_ssm.h")


@pytest.fixture(scope="module")
def lib():
    lib_build.build()
    return m.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mamba_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("mamba_selective_scan", "mamba_selective_scan_ex", "mamba_state_update",
                 "mamba_status_string", "mamba_get_device_error"):
        assert want in names


def test_library_exports_every_declared_function(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/mamba_ssm.h but not exported"
    # and the binding wraps each of them under the same name
    for name in declared_functions():
        assert hasattr(m, name), f"binding lacks {name}"


def test_status_strings(lib):
    assert m.status_string(m.MAMBA_OK) == "ok"
    assert "invalid" in m.status_string(m.MAMBA_ERR_INVALID_ARG)
    assert "timed out" in m.status_string(m.MAMBA_ERR_TIMEOUT)
    assert m.status_string(12345) == "unknown status"


def test_supported_nstate(lib):
    for n in (4, 8, 16, 32):
        assert m.mamba_scan_supported_nstate(n)
    for n in (0, 1, 2, 12, 17, 64):
        assert not m.mamba_scan_supported_nstate(n)


def _scan_ex(lib, **kw):
    a = dict(u=1024, delta=1024, A=1024, B=1024, C=1024, D=None, h0=None, y=2048, fs=None, batch=1, len=4,
             channels=8, nstate=16, chunk=0, flags=0, dtype=m.MAMBA_BF16)
    a.update(kw)
    return lib.mamba_selective_scan_ex(a["u"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["h0"], a["y"],
                                       a["fs"], a["batch"], a["len"], a["channels"], a["nstate"], a["chunk"],
                                       a["flags"], a["dtype"], None)


def test_scan_argument_errors_on_host(lib):
    # every case below is rejected before any CUDA call is made
    assert _scan_ex(lib, dtype=7) == m.MAMBA_ERR_INVALID_ARG
    assert _scan_ex(lib, batch=-1) == m.MAMBA_ERR_INVALID_ARG
    assert _scan_ex(lib, len=-3) == m.MAMBA_ERR_INVALID_ARG
    assert _scan_ex(lib, channels=-1) == m.MAMBA_ERR_INVALID_ARG
    assert _scan_ex(lib, chunk=-1) == m.MAMBA_ERR_INVALID_ARG
    assert _scan_ex(lib, flags=8) == m.MAMBA_ERR_INVALID_ARG
    assert _scan_ex(lib, flags=m.MAMBA_SCAN_EULER | m.MAMBA_SCAN_TRAPEZOID) == m.MAMBA_ERR_INVALID_ARG
    assert _scan_ex(lib, nstate=0) == m.MAMBA_ERR_INVALID_ARG
    assert _scan_ex(lib, nstate=12) == m.MAMBA_ERR_UNSUPPORTED
    assert _scan_ex(lib, u=None) == m.MAMBA_ERR_INVALID_ARG
    assert _scan_ex(lib, y=None) == m.MAMBA_ERR_INVALID_ARG
    assert _scan_ex(lib, A=None) == m.MAMBA_ERR_INVALID_ARG
    assert _scan_ex(lib, u=1025) == m.MAMBA_ERR_INVALID_ARG            # misaligned bf16 pointer
    assert _scan_ex(lib, dtype=m.MAMBA_F32, u=1026) == m.MAMBA_ERR_INVALID_ARG
    assert _scan_ex(lib, batch=1 << 20, len=1 << 12) == m.MAMBA_ERR_UNSUPPORTED   # batch*len >= 2^31
    # empty problems are valid no-ops
    assert _scan_ex(lib, batch=0) == m.MAMBA_OK
    assert _scan_ex(lib, channels=0) == m.MAMBA_OK
    assert _scan_ex(lib, len=0, fs=None) == m.MAMBA_OK


def _ssd(lib, **kw):
    a = dict(x=1024, dt=1024, A=1024, B=1024, C=1024, D=None, h0=None, y=2048, fs=None, batch=1, len=4,
             heads=2, headdim=64, nstate=16, supers=0, flags=0, dtype=m.MAMBA_BF16)
    a.update(kw)
    return lib.mamba_ssd_scan(a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"], a["h0"], a["y"], a["fs"],
                              a["batch"], a["len"], a["heads"], a["headdim"], a["nstate"], a["supers"],
                              a["flags"], a["dtype"], None)


def test_ssd_argument_errors_on_host(lib):
    # every case below is rejected (or is a no-op) before any CUDA call is made
    assert _ssd(lib, dtype=7) == m.MAMBA_ERR_INVALID_ARG
    assert _ssd(lib, batch=-1) == m.MAMBA_ERR_INVALID_ARG
    assert _ssd(lib, len=-1) == m.MAMBA_ERR_INVALID_ARG
    assert _ssd(lib, heads=-1) == m.MAMBA_ERR_INVALID_ARG
    assert _ssd(lib, headdim=0) == m.MAMBA_ERR_INVALID_ARG
    assert _ssd(lib, supers=-1) == m.MAMBA_ERR_INVALID_ARG
    assert _ssd(lib, flags=8) == m.MAMBA_ERR_INVALID_ARG
    assert _ssd(lib, flags=m.MAMBA_SCAN_EULER | m.MAMBA_SCAN_TRAPEZOID) == m.MAMBA_ERR_INVALID_ARG
    assert _ssd(lib, flags=m.MAMBA_SCAN_TRAPEZOID) == m.MAMBA_ERR_UNSUPPORTED
    assert _ssd(lib, dtype=m.MAMBA_F32) == m.MAMBA_ERR_UNSUPPORTED
    assert _ssd(lib, headdim=32) == m.MAMBA_ERR_UNSUPPORTED
    for n in (4, 8, 12, 128):
        assert _ssd(lib, nstate=n) == m.MAMBA_ERR_UNSUPPORTED
    for n in (16, 32, 64):
        assert m.mamba_ssd_supported_nstate(n)
    assert _ssd(lib, x=None) == m.MAMBA_ERR_INVALID_ARG
    assert _ssd(lib, dt=None) == m.MAMBA_ERR_INVALID_ARG
    assert _ssd(lib, y=None) == m.MAMBA_ERR_INVALID_ARG
    assert _ssd(lib, x=1032) == m.MAMBA_ERR_INVALID_ARG          # x not 16-byte aligned
    assert _ssd(lib, B=1040 + 2) == m.MAMBA_ERR_INVALID_ARG
    assert _ssd(lib, y=2056) == m.MAMBA_ERR_INVALID_ARG
    assert _ssd(lib, dt=1025) == m.MAMBA_ERR_INVALID_ARG
    assert _ssd(lib, D=1028) == m.MAMBA_ERR_INVALID_ARG          # D not 8-byte aligned
    assert _ssd(lib, batch=1 << 20, len=1 << 12) == m.MAMBA_ERR_UNSUPPORTED
    assert _ssd(lib, batch=0) == m.MAMBA_OK
    assert _ssd(lib, heads=0) == m.MAMBA_OK
    assert _ssd(lib, len=0, fs=None) == m.MAMBA_OK


def _cplx(lib, **kw):
    a = dict(u=1024, delta=1024, Are=1024, Aim=1024, B=1024, C=1024, D=None, h0=None, y=2048, fs=None, batch=1,
             len=4, channels=8, nstate=16, supers=0, dtype=m.MAMBA_BF16)
    a.update(kw)
    return lib.mamba_selective_scan_complex(a["u"], a["delta"], a["Are"], a["Aim"], a["B"], a["C"], a["D"],
                                            a["h0"], a["y"], a["fs"], a["batch"], a["len"], a["channels"],
                                            a["nstate"], a["supers"], a["dtype"], None)


def test_complex_scan_argument_errors_on_host(lib):
    assert _cplx(lib, dtype=7) == m.MAMBA_ERR_INVALID_ARG
    assert _cplx(lib, batch=-1) == m.MAMBA_ERR_INVALID_ARG
    assert _cplx(lib, len=-1) == m.MAMBA_ERR_INVALID_ARG
    assert _cplx(lib, channels=-1) == m.MAMBA_ERR_INVALID_ARG
    assert _cplx(lib, supers=-1) == m.MAMBA_ERR_INVALID_ARG
    for n in (2, 12, 32):
        assert _cplx(lib, nstate=n) == m.MAMBA_ERR_UNSUPPORTED
    for n in (4, 8, 16):
        assert m.mamba_complex_supported_nstate(n)
    assert _cplx(lib, Aim=None) == m.MAMBA_ERR_INVALID_ARG
    assert _cplx(lib, u=None) == m.MAMBA_ERR_INVALID_ARG
    assert _cplx(lib, u=1025) == m.MAMBA_ERR_INVALID_ARG
    assert _cplx(lib, dtype=m.MAMBA_F32, B=1026) == m.MAMBA_ERR_INVALID_ARG
    assert _cplx(lib, h0=1028) == m.MAMBA_ERR_INVALID_ARG          # complex state: 8-byte aligned
    assert _cplx(lib, batch=1 << 20, len=1 << 12) == m.MAMBA_ERR_UNSUPPORTED
    assert _cplx(lib, batch=0) == m.MAMBA_OK
    assert _cplx(lib, channels=0) == m.MAMBA_OK
    assert _cplx(lib, len=0, fs=None) == m.MAMBA_OK


def test_state_update_argument_errors_on_host(lib):
    f = lib.mamba_state_update
    ok = dict(state=4096, x=1024, delta=1024, A=4096, B=1024, C=1024, D=None, y=2048, batch=2, channels=8,
              nstate=16, dtype=m.MAMBA_BF16)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["state"], a["x"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["y"], a["batch"],
                 a["channels"], a["nstate"], a["dtype"], None)

    assert call(dtype=3) == m.MAMBA_ERR_INVALID_ARG
    assert call(batch=-2) == m.MAMBA_ERR_INVALID_ARG
    assert call(nstate=12) == m.MAMBA_ERR_UNSUPPORTED
    assert call(state=None) == m.MAMBA_ERR_INVALID_ARG
    assert call(state=4100) == m.MAMBA_ERR_INVALID_ARG                   # state must be 16-byte aligned
    assert call(B=1026) == m.MAMBA_ERR_INVALID_ARG
    assert call(batch=0) == m.MAMBA_OK


def test_host_scan_argument_errors(lib):
    # rejected on the host before any CUDA call
    f = lib.mamba_selective_scan_host
    args = [1024, 1024, 1024, 1024, 1024, None, 2048, None, 1, 4, 8, 16, 0, m.MAMBA_BF16, None]
    def call(i, v):
        a = list(args)
        a[i] = v
        return f(*a)
    assert call(13, 5) == m.MAMBA_ERR_INVALID_ARG       # dtype
    assert call(8, -1) == m.MAMBA_ERR_INVALID_ARG       # batch
    assert call(12, -1) == m.MAMBA_ERR_INVALID_ARG      # piece_len
    assert call(11, 12) == m.MAMBA_ERR_UNSUPPORTED      # nstate
    assert call(2, None) == m.MAMBA_ERR_INVALID_ARG     # A
    assert call(0, None) == m.MAMBA_ERR_INVALID_ARG     # u
    assert call(8, 0) == m.MAMBA_OK                     # empty


def test_backward_argument_errors(lib):
    f = lib.mamba_selective_scan_backward
    base = [1024] * 16 + [1, 4, 8, 16, m.MAMBA_BF16, None]
    base[5] = None   # D
    base[6] = None   # initial state
    base[8] = None   # d_final_state
    base[14] = None  # dD
    base[15] = None  # d_initial_state

    def call(i, v):
        a = list(base)
        a[i] = v
        return f(*a)
    assert call(20, 9) == m.MAMBA_ERR_INVALID_ARG      # dtype
    assert call(16, -1) == m.MAMBA_ERR_INVALID_ARG     # batch
    assert call(19, 12) == m.MAMBA_ERR_UNSUPPORTED     # nstate
    assert call(19, 32) == m.MAMBA_ERR_UNSUPPORTED     # nstate 32: forward only
    assert call(7, None) == m.MAMBA_ERR_INVALID_ARG    # dy
    assert call(11, None) == m.MAMBA_ERR_INVALID_ARG   # dA
    assert call(5, 1024) == m.MAMBA_ERR_INVALID_ARG    # D given without dD
    assert call(9, 1025) == m.MAMBA_ERR_INVALID_ARG    # misaligned du
    assert call(16, 0) == m.MAMBA_OK                   # empty


def test_library_links_no_torch(lib):
    # the product library is plain C ABI over CUDA: no torch / python symbols needed
    out = os.popen(f"nm -D --undefined-only {lib_build.LIB}").read()
    assert "torch" not in out and "Py" not in out


def test_scan_plan_host_logic(lib):
    """The planner (host only when the SM count is given): enough parallel
    streams for 4 warps per SM, jobs that cover the sequence, and the
    super-chunk split only when groups are scarce."""
    sms = 148
    # mid workload: 8 x 3072 channels = 768 groups >= 592 warps -> no split
    p = m.mamba_scan_plan(8, 2048, 3072, 16, 0, m.MAMBA_BF16, sms)
    assert p.supers == 1 and p.kernels == 2 and p.consumer_warps == 4
    assert p.jobs * p.chunk_len >= 768 * 2048 and p.jobs >= 8 * 592 * 0.9
    assert p.ctas == sms
    # long workload: 64 groups -> split into super-chunks that run from zero
    # side by side; pre-pass, chunked kernel, correction kernel.  The
    # super-chunks are long, so the CTAs carry eight consumer warps
    p = m.mamba_scan_plan(1, 1 << 20, 2048, 16, 0, m.MAMBA_BF16, sms)
    assert p.supers > 1 and p.kernels == 3 and p.consumer_warps == 8
    assert p.supers * 64 >= sms * 8
    assert p.super_len * p.supers >= 1 << 20 and p.super_len * (p.supers - 1) < 1 << 20
    # every job is a chunk of a main stream: the jobs cover each stream once
    assert p.jobs * p.chunk_len >= 64 * (1 << 20) and (p.jobs - 64 * p.supers) * p.chunk_len < 64 * (1 << 20)
    # shorter super-chunks, other state counts and forced chunking keep four
    assert m.mamba_scan_plan(1, 1 << 19, 2048, 16, 0, m.MAMBA_BF16, sms).consumer_warps == 4
    assert m.mamba_scan_plan(1, 1 << 20, 2048, 16, 0, m.MAMBA_F32, sms).consumer_warps == 4
    assert m.mamba_scan_plan(1, 1 << 20, 2048, 32, 0, m.MAMBA_BF16, sms).consumer_warps == 4
    assert m.mamba_scan_plan(1, 1 << 20, 2048, 16, 4096, m.MAMBA_BF16, sms).consumer_warps == 4
    # forced chunking
    p = m.mamba_scan_plan(2, 1000, 200, 16, 37, m.MAMBA_BF16, sms)
    assert p.super_len == 37 and p.supers == 28 and p.kernels == 3
    # tiny problem: one CTA per four jobs
    p = m.mamba_scan_plan(1, 10, 32, 16, 0, m.MAMBA_F32, sms)
    assert p.supers == 1 and p.jobs == 1 and p.ctas == 1
    assert p.scratch_bytes > 0
    # empty problem: nothing planned
    p = m.mamba_scan_plan(1, 0, 32, 16, 0, m.MAMBA_F32, sms)
    assert p.kernels == 0
    with pytest.raises(m.MambaError):
        m.mamba_scan_plan(1, 10, 32, 12, 0, m.MAMBA_F32, sms)

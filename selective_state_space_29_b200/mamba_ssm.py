"""Python binding of the C ABI in include/mamba_ssm.h (argument marshalling only).

Every function named like a C entry point forwards its arguments to the
library unchanged: tensors become device pointers, torch streams become
`cudaStream_t` handles, a non-zero status raises `MambaError`.  The
tensor-level helpers (`selective_scan`, `ssd_scan`, `state_update`, ...) only allocate the
outputs with torch and then make the same C calls.  There is no fallback: if
the library is missing or cannot load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libmamba_ssm_b200.so")

MAMBA_F32 = 0
MAMBA_BF16 = 1
MAMBA_OK = 0
MAMBA_ERR_INVALID_ARG = 1
MAMBA_ERR_UNSUPPORTED = 2
MAMBA_ERR_CUDA = 3
MAMBA_ERR_TIMEOUT = 4
MAMBA_SCAN_GENERAL_A = 1
MAMBA_SCAN_EULER = 2
MAMBA_SCAN_TRAPEZOID = 4

class ScanPlan(ctypes.Structure):
    """mamba_scan_plan_t"""
    _fields_ = [("supers", ctypes.c_int64), ("super_len", ctypes.c_int64), ("chunk_len", ctypes.c_int64),
                ("jobs", ctypes.c_int64), ("kernels", ctypes.c_int64), ("scratch_bytes", ctypes.c_int64),
                ("ctas", ctypes.c_int64), ("consumer_warps", ctypes.c_int64)]

    def as_dict(self):
        return {k: int(getattr(self, k)) for k, _ in self._fields_}


# (name, restype, argtypes) for every entry point of include/mamba_ssm.h
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SIGNATURES = [
    ("mamba_selective_scan", ctypes.c_int,
     [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, ctypes.c_int, _P]),
    ("mamba_selective_scan_ex", ctypes.c_int,
     [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, ctypes.c_uint, ctypes.c_int, _P]),
    ("mamba_selective_scan_noalloc", ctypes.c_int,
     [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, ctypes.c_int, _P]),
    ("mamba_selective_scan_host", ctypes.c_int,
     [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int, _P]),
    ("mamba_selective_scan_backward", ctypes.c_int,
     [_P] * 16 + [_I64, _I64, _I64, _I64, ctypes.c_int, _P]),
    ("mamba_state_update", ctypes.c_int,
     [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, ctypes.c_int, _P]),
    ("mamba_ssd_scan", ctypes.c_int,
     [_P] * 9 + [_I64] * 6 + [ctypes.c_uint, ctypes.c_int, _P]),
    ("mamba_ssd_supported_nstate", ctypes.c_int, [_I64]),
    ("mamba_selective_scan_complex", ctypes.c_int,
     [_P] * 10 + [_I64] * 5 + [ctypes.c_int, _P]),
    ("mamba_complex_supported_nstate", ctypes.c_int, [_I64]),
    ("mamba_selective_scan_mimo", ctypes.c_int,
     [_P] * 9 + [_I64] * 5 + [ctypes.c_uint, ctypes.c_int, _P]),
    ("mamba_mimo_supported", ctypes.c_int, [_I64, _I64]),
    ("mamba_state_update_mimo", ctypes.c_int,
     [_P] * 8 + [_I64] * 4 + [ctypes.c_int, _P]),
    ("mamba_scan_plan", ctypes.c_int,
     [_I64, _I64, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ScanPlan)]),
    ("mamba_status_string", ctypes.c_char_p, [ctypes.c_int]),
    ("mamba_scan_supported_nstate", ctypes.c_int, [_I64]),
    ("mamba_get_device_error", ctypes.c_int, [_P, ctypes.c_int]),
    ("mamba_debug_scratch_allocations", ctypes.c_int64, []),
    ("mamba_trim_scratch_pool", ctypes.c_int, []),
    ("mamba_debug_expire_wait", ctypes.c_int, [_I64, _P]),
]


class MambaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None


def library() -> ctypes.CDLL:
    """Load libmamba_ssm_b200.so (built by `python -m selective_state_space_29_b200.build`)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m selective_state_space_29_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, res, args in _SIGNATURES:
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return library().mamba_status_string(int(status)).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, what: str):
    if status != MAMBA_OK:
        raise MambaError(status, what)


def dtype_code(torch_dtype) -> int:
    import torch
    if torch_dtype == torch.float32:
        return MAMBA_F32
    if torch_dtype == torch.bfloat16:
        return MAMBA_BF16
    raise ValueError(f"unsupported dtype {torch_dtype}")


# --- the C entry points -------------------------------------------------------

def mamba_selective_scan(u, delta, A, B, C, D, y, final_state, batch, len, channels, nstate, dtype,
                         stream=None):
    st = library().mamba_selective_scan(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(y),
                                        _ptr(final_state), batch, len, channels, nstate, dtype,
                                        _stream(stream))
    _check(st, "mamba_selective_scan")


def mamba_selective_scan_ex(u, delta, A, B, C, D, initial_state, y, final_state, batch, len, channels, nstate,
                            chunk_len, flags, dtype, stream=None):
    st = library().mamba_selective_scan_ex(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                           _ptr(initial_state), _ptr(y), _ptr(final_state), batch, len,
                                           channels, nstate, chunk_len, flags, dtype, _stream(stream))
    _check(st, "mamba_selective_scan_ex")


def mamba_selective_scan_noalloc(u, delta, A, B, C, D, y, final_state, batch, len, channels, nstate, dtype,
                                 stream=None):
    """The scan with its scratch in the library's fixed 16 MiB device array:
    no device allocation, for callers that may not allocate inside an
    operation.  Calls that overlap on the GPU race on that array."""
    st = library().mamba_selective_scan_noalloc(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(y),
                                                _ptr(final_state), batch, len, channels, nstate, dtype,
                                                _stream(stream))
    _check(st, "mamba_selective_scan_noalloc")


def mamba_selective_scan_host(u, delta, A, B, C, D, y, final_state, batch, len, channels, nstate, piece_len,
                              dtype, stream=None):
    """The scan on host buffers (page-locked for overlap), copies pipelined
    with the scan piece by piece; asynchronous on `stream`."""
    st = library().mamba_selective_scan_host(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(y),
                                             _ptr(final_state), batch, len, channels, nstate, piece_len, dtype,
                                             _stream(stream))
    _check(st, "mamba_selective_scan_host")


def mamba_selective_scan_backward(u, delta, A, B, C, D, initial_state, dy, d_final_state, du, ddelta, dA, dB, dC,
                                  dD, d_initial_state, batch, len, channels, nstate, dtype, stream=None):
    st = library().mamba_selective_scan_backward(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(initial_state), _ptr(dy), _ptr(d_final_state),
        _ptr(du), _ptr(ddelta), _ptr(dA), _ptr(dB), _ptr(dC), _ptr(dD), _ptr(d_initial_state), batch, len, channels,
        nstate, dtype, _stream(stream))
    _check(st, "mamba_selective_scan_backward")


def mamba_state_update(state, x, delta, A, B, C, D, y, batch, channels, nstate, dtype, stream=None):
    st = library().mamba_state_update(_ptr(state), _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                      _ptr(y), batch, channels, nstate, dtype, _stream(stream))
    _check(st, "mamba_state_update")


def mamba_ssd_scan(x, dt, A, B, C, D, initial_state, y, final_state, batch, len, heads, headdim, nstate, supers,
                   flags, dtype, stream=None):
    st = library().mamba_ssd_scan(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(initial_state),
                                  _ptr(y), _ptr(final_state), batch, len, heads, headdim, nstate, supers, flags,
                                  dtype, _stream(stream))
    _check(st, "mamba_ssd_scan")


def mamba_ssd_supported_nstate(nstate: int) -> bool:
    return bool(library().mamba_ssd_supported_nstate(int(nstate)))


def mamba_selective_scan_complex(u, delta, A_re, A_im, B, C, D, initial_state, y, final_state, batch, len, channels,
                                 nstate, supers, dtype, stream=None):
    st = library().mamba_selective_scan_complex(_ptr(u), _ptr(delta), _ptr(A_re), _ptr(A_im), _ptr(B), _ptr(C),
                                                _ptr(D), _ptr(initial_state), _ptr(y), _ptr(final_state), batch, len,
                                                channels, nstate, supers, dtype, _stream(stream))
    _check(st, "mamba_selective_scan_complex")


def mamba_complex_supported_nstate(nstate: int) -> bool:
    return bool(library().mamba_complex_supported_nstate(int(nstate)))


def mamba_selective_scan_mimo(u, delta, A, B, C, D, initial_state, y, final_state, batch, len, ranks, channels,
                              nstate, flags, dtype, stream=None):
    st = library().mamba_selective_scan_mimo(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                             _ptr(initial_state), _ptr(y), _ptr(final_state), batch, len, ranks,
                                             channels, nstate, flags, dtype, _stream(stream))
    _check(st, "mamba_selective_scan_mimo")


def mamba_state_update_mimo(state, x, delta, A, B, C, D, y, batch, ranks, channels, nstate, dtype, stream=None):
    st = library().mamba_state_update_mimo(_ptr(state), _ptr(x), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                           _ptr(y), batch, ranks, channels, nstate, dtype, _stream(stream))
    _check(st, "mamba_state_update_mimo")


def mamba_mimo_supported(ranks: int, nstate: int) -> bool:
    return bool(library().mamba_mimo_supported(int(ranks), int(nstate)))


def mamba_scan_plan(batch, len, channels, nstate, chunk_len, dtype, sm_count=0) -> ScanPlan:
    out = ScanPlan()
    _check(library().mamba_scan_plan(batch, len, channels, nstate, chunk_len, dtype, sm_count,
                                     ctypes.byref(out)), "mamba_scan_plan")
    return out


def mamba_status_string(status: int) -> str:
    return status_string(status)


def mamba_scan_supported_nstate(nstate: int) -> bool:
    return bool(library().mamba_scan_supported_nstate(int(nstate)))


def mamba_get_device_error(clear: bool = False, stream=None) -> int:
    return int(library().mamba_get_device_error(_stream(stream), 1 if clear else 0))


def mamba_debug_scratch_allocations() -> int:
    return int(library().mamba_debug_scratch_allocations())


def mamba_trim_scratch_pool():
    _check(library().mamba_trim_scratch_pool(), "mamba_trim_scratch_pool")


def mamba_debug_expire_wait(limit_ns: int, stream=None):
    _check(library().mamba_debug_expire_wait(int(limit_ns), _stream(stream)), "mamba_debug_expire_wait")


# --- tensor-level helpers ---------------------------------------------------------

_METHOD_FLAGS = {"zoh": 0, "euler": MAMBA_SCAN_EULER, "trapezoid": MAMBA_SCAN_TRAPEZOID}


def selective_scan(u, delta, A, B, C, D=None, initial_state=None, return_final_state=True, chunk_len=0,
                   general_a=False, y=None, final_state=None, stream=None, method="zoh"):
    """y, final_state = selective_scan(u, delta, A, B, C, D) on CUDA tensors.

    u, delta: (batch, len, channels); B, C: (batch, len, nstate) of one dtype
    (float32 or bfloat16); A: (channels, nstate) float32; D: (channels,) or
    None; initial_state: (batch, channels, nstate) float32 or None; method:
    "zoh" (default), "euler" or "trapezoid" (see MAMBA_SCAN_EULER)."""
    import torch
    batch, length, channels = u.shape
    nstate = A.shape[1]
    for t in (u, delta, A, B, C, D, initial_state):
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    if y is None:
        y = torch.empty_like(u)
    if final_state is None and return_final_state:
        final_state = torch.empty((batch, channels, nstate), device=u.device, dtype=torch.float32)
    flags = (MAMBA_SCAN_GENERAL_A if general_a else 0) | _METHOD_FLAGS[method]
    if initial_state is None and chunk_len == 0 and flags == 0:
        mamba_selective_scan(u, delta, A, B, C, D, y, final_state, batch, length, channels, nstate,
                             dtype_code(u.dtype), stream)
    else:
        mamba_selective_scan_ex(u, delta, A, B, C, D, initial_state, y, final_state, batch, length, channels,
                                nstate, chunk_len, flags, dtype_code(u.dtype), stream)
    return y, final_state


def state_update(state, x, delta, A, B, C, D=None, y=None, stream=None):
    """One recurrent step in place on `state` (batch, channels, nstate) float32;
    returns y (batch, channels) in the dtype of x."""
    import torch
    batch, channels, nstate = state.shape
    if y is None:
        y = torch.empty_like(x)
    mamba_state_update(state, x, delta, A, B, C, D, y, batch, channels, nstate, dtype_code(x.dtype), stream)
    return y


def ssd_scan(x, dt, A, B, C, D=None, initial_state=None, return_final_state=True, headdim=64, supers=0,
             method="zoh", y=None, final_state=None, stream=None):
    """y, final_state = Mamba-2's scalar-A scan on CUDA tensors.

    x: (batch, len, heads*headdim) bfloat16; dt: (batch, len, heads)
    bfloat16; A: (heads,) float32; B, C: (batch, len, nstate) bfloat16; D:
    (heads*headdim,) float32 or None; initial_state: (batch,
    heads*headdim, nstate) float32 or None; method "zoh" or "euler"."""
    import torch
    batch, length, channels = x.shape
    heads = A.shape[0]
    nstate = B.shape[2]
    for t in (x, dt, A, B, C, D, initial_state):
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    if channels != heads * headdim:
        raise ValueError("x must have heads*headdim channels")
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and return_final_state:
        final_state = torch.empty((batch, channels, nstate), device=x.device, dtype=torch.float32)
    mamba_ssd_scan(x, dt, A, B, C, D, initial_state, y, final_state, batch, length, heads, headdim, nstate, supers,
                   _METHOD_FLAGS[method], dtype_code(x.dtype), stream)
    return y, final_state


def selective_scan_complex(u, delta, A_re, A_im, B, C, D=None, initial_state=None, return_final_state=True,
                           supers=0, y=None, final_state=None, stream=None):
    """y, final_state = the scan with a complex diagonal A = A_re + i A_im.

    u, delta: (batch, len, channels); B, C: (batch, len, nstate) of one dtype
    (float32 or bfloat16); A_re, A_im: (channels, nstate) float32; D:
    (channels,) or None; initial_state and the returned final state:
    (batch, channels, nstate, 2) float32, (re, im) in the last index."""
    import torch
    batch, length, channels = u.shape
    nstate = A_re.shape[1]
    for t in (u, delta, A_re, A_im, B, C, D, initial_state):
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    if y is None:
        y = torch.empty_like(u)
    if final_state is None and return_final_state:
        final_state = torch.empty((batch, channels, nstate, 2), device=u.device, dtype=torch.float32)
    mamba_selective_scan_complex(u, delta, A_re, A_im, B, C, D, initial_state, y, final_state, batch, length,
                                 channels, nstate, supers, dtype_code(u.dtype), stream)
    return y, final_state


def selective_scan_host(u, delta, A, B, C, D=None, y=None, final_state=None, piece_len=0, stream=None,
                        synchronize=True):
    """y, final_state = the scan of host tensors (CPU, ideally pinned), with
    the host<->device copies overlapped with the scan; outputs are host
    tensors (allocated pinned when not given)."""
    import torch
    batch, length, channels = u.shape
    nstate = A.shape[1]
    for t in (u, delta, A, B, C, D):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError("host tensors must be contiguous CPU tensors")
    if y is None:
        y = torch.empty(u.shape, dtype=u.dtype, pin_memory=True)
    if final_state is None:
        final_state = torch.empty((batch, channels, nstate), dtype=torch.float32, pin_memory=True)
    mamba_selective_scan_host(u, delta, A, B, C, D, y, final_state, batch, length, channels, nstate, piece_len,
                              dtype_code(u.dtype), stream)
    if synchronize:
        torch.cuda.synchronize()
    return y, final_state


def selective_scan_backward(u, delta, A, B, C, D, dy, initial_state=None, d_final_state=None, stream=None):
    """Gradients of the zero-order-hold scan for an upstream gradient dy of y
    (and d_final_state of the final state), on CUDA tensors.  Returns a dict:
    du, ddelta (dtype of u), dA, dB, dC, dD (None without D), d_initial_state
    (float32)."""
    import torch
    batch, length, channels = u.shape
    nstate = A.shape[1]
    for t in (u, delta, A, B, C, D, dy, initial_state, d_final_state):
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    f32 = dict(device=u.device, dtype=torch.float32)
    out = {"du": torch.empty_like(u), "ddelta": torch.empty_like(delta), "dA": torch.empty(A.shape, **f32),
           "dB": torch.empty(B.shape, **f32), "dC": torch.empty(C.shape, **f32),
           "dD": None if D is None else torch.empty(D.shape, **f32),
           "d_initial_state": torch.empty((batch, channels, nstate), **f32)}
    mamba_selective_scan_backward(u, delta, A, B, C, D, initial_state, dy, d_final_state, out["du"], out["ddelta"],
                                  out["dA"], out["dB"], out["dC"], out["dD"], out["d_initial_state"], batch, length,
                                  channels, nstate, dtype_code(u.dtype), stream)
    return out


def selective_scan_mimo(u, delta, A, B, C, D=None, initial_state=None, return_final_state=True, general_a=False,
                        y=None, final_state=None, stream=None):
    """y, final_state = selective_scan_mimo(u, delta, A, B, C, D) on CUDA tensors.

    u: (batch, len, ranks, channels); delta: (batch, len, channels); B, C:
    (batch, len, ranks, nstate), one dtype (float32 or bfloat16); A:
    (channels, nstate) float32; D: (channels,) or None; initial_state:
    (batch, channels, nstate) float32 or None.  y is shaped like u."""
    import torch
    batch, length, ranks, channels = u.shape
    nstate = A.shape[1]
    for t in (u, delta, A, B, C, D, initial_state):
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    if y is None:
        y = torch.empty_like(u)
    if final_state is None and return_final_state:
        final_state = torch.empty((batch, channels, nstate), device=u.device, dtype=torch.float32)
    mamba_selective_scan_mimo(u, delta, A, B, C, D, initial_state, y, final_state, batch, length, ranks, channels,
                              nstate, MAMBA_SCAN_GENERAL_A if general_a else 0, dtype_code(u.dtype), stream)
    return y, final_state


def state_update_mimo(state, x, delta, A, B, C, D=None, y=None, stream=None):
    """One multi-input multi-output recurrent step, state updated in place.
    state: (batch, channels, nstate) float32; x: (batch, ranks, channels);
    delta: (batch, channels); B, C: (batch, ranks, nstate).  Returns y, shaped like x."""
    import torch
    batch, ranks, channels = x.shape
    nstate = A.shape[1]
    if y is None:
        y = torch.empty_like(x)
    mamba_state_update_mimo(state, x, delta, A, B, C, D, y, batch, ranks, channels, nstate, dtype_code(x.dtype), stream)
    return y

"""fp64 CPU oracle for the selective scan and the recurrent state update.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
benchmark's CPU-baseline leg, never by the product library.  The arithmetic
lives in `ssm_oracle.c` (plain C, double precision); this module only moves
numpy arrays across ctypes.  It follows the zero-order-hold discretisation and
recurrence of "Mamba SSM Nedir? Transformer Alternatifi Rehberi (2026)",
sections "State Space Model Temelleri" and "Ayrık Zamana Geçiş", and, as
options, the exponential-Euler and trapezoidal discretisations that the
Mamba-3 page names in "Geliştirilmiş Ayrıklaştırma Şeması"; also the
complex-valued and the multi-input multi-output (MIMO) state of that page.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_c_f64p = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


class Oracle:
    """One loaded copy of the oracle library (a test may load a modified copy)."""

    def __init__(self, lib_path: str | None = None):
        path = lib_path or _build.build()
        self.path = path
        self._lib = ctypes.CDLL(os.path.abspath(path))
        self._lib.oracle_scan.restype = ctypes.c_int
        self._lib.oracle_scan.argtypes = [_c_f64p] * 9 + [_i64] * 4 + [ctypes.c_int]
        self._lib.oracle_scan_method.restype = ctypes.c_int
        self._lib.oracle_scan_method.argtypes = [_c_f64p] * 9 + [_i64] * 4 + [ctypes.c_int, ctypes.c_int]
        self._lib.oracle_scan_backward.restype = ctypes.c_int
        self._lib.oracle_scan_backward.argtypes = [_c_f64p] * 16 + [_i64] * 4
        self._lib.oracle_state_update.restype = ctypes.c_int
        self._lib.oracle_state_update.argtypes = [_c_f64p] * 8 + [_i64] * 3 + [ctypes.c_int]
        self._lib.oracle_scan_complex.restype = ctypes.c_int
        self._lib.oracle_scan_complex.argtypes = [_c_f64p] * 10 + [_i64] * 4 + [ctypes.c_int]
        self._lib.oracle_scan_mimo.restype = ctypes.c_int
        self._lib.oracle_scan_mimo.argtypes = [_c_f64p] * 9 + [_i64] * 5 + [ctypes.c_int]
        self._lib.oracle_max_threads.restype = ctypes.c_int

    @staticmethod
    def _ptr(a):
        return None if a is None else a.ctypes.data_as(_c_f64p)

    @staticmethod
    def _f64(a):
        return None if a is None else np.ascontiguousarray(np.asarray(a, dtype=np.float64))

    # discretisations (oracle_scan_method): zero-order hold, exponential
    # Euler, trapezoidal -- see ssm_oracle.c for the readings
    ZOH, EULER, TRAPEZOID = 0, 1, 2

    def scan(self, u, delta, A, B, C, D=None, h0=None, want_y=True, nthreads=0, method=0):
        """Selective scan.  u, delta: (batch, len, channels); B, C: (batch, len,
        nstate); A: (channels, nstate); D: (channels,) or None; h0: (batch,
        channels, nstate) or None; method: ZOH, EULER or TRAPEZOID.  Returns
        (y, h_final) in float64."""
        u, delta, A, B, C, D, h0 = map(self._f64, (u, delta, A, B, C, D, h0))
        batch, length, channels = u.shape
        nstate = A.shape[1]
        assert delta.shape == u.shape and A.shape == (channels, nstate)
        assert B.shape == (batch, length, nstate) and C.shape == B.shape
        assert D is None or D.shape == (channels,)
        assert h0 is None or h0.shape == (batch, channels, nstate)
        y = np.empty_like(u) if want_y else None
        hf = np.empty((batch, channels, nstate), dtype=np.float64)
        if method == self.ZOH:
            rc = self._lib.oracle_scan(self._ptr(u), self._ptr(delta), self._ptr(A), self._ptr(B),
                                       self._ptr(C), self._ptr(D), self._ptr(h0), self._ptr(y),
                                       self._ptr(hf), batch, length, channels, nstate, int(nthreads))
        else:
            rc = self._lib.oracle_scan_method(self._ptr(u), self._ptr(delta), self._ptr(A), self._ptr(B),
                                              self._ptr(C), self._ptr(D), self._ptr(h0), self._ptr(y),
                                              self._ptr(hf), batch, length, channels, nstate, int(method),
                                              int(nthreads))
        if rc != 0:
            raise RuntimeError(f"oracle_scan failed ({rc})")
        return y, hf

    def scan_backward(self, u, delta, A, B, C, D, dy, h0=None, dh_final=None):
        """Gradients of the zero-order-hold scan for an upstream gradient dy of
        y (and dh_final of the final state): returns a dict with du, ddelta,
        dA, dB, dC, dD (None when D is None) and dh0, all float64."""
        u, delta, A, B, C, D, dy, h0, dh_final = map(self._f64, (u, delta, A, B, C, D, dy, h0, dh_final))
        batch, length, channels = u.shape
        nstate = A.shape[1]
        assert dy.shape == u.shape
        out = {"du": np.empty_like(u), "ddelta": np.empty_like(u), "dA": np.empty_like(A),
               "dB": np.empty_like(B), "dC": np.empty_like(C),
               "dD": None if D is None else np.empty_like(D),
               "dh0": np.empty((batch, channels, nstate), dtype=np.float64)}
        rc = self._lib.oracle_scan_backward(
            self._ptr(u), self._ptr(delta), self._ptr(A), self._ptr(B), self._ptr(C), self._ptr(D), self._ptr(h0),
            self._ptr(dy), self._ptr(dh_final), self._ptr(out["du"]), self._ptr(out["ddelta"]), self._ptr(out["dA"]),
            self._ptr(out["dB"]), self._ptr(out["dC"]), self._ptr(out["dD"]), self._ptr(out["dh0"]),
            batch, length, channels, nstate)
        if rc != 0:
            raise RuntimeError(f"oracle_scan_backward failed ({rc})")
        return out

    def state_update(self, state, x, delta, A, B, C, D=None, nthreads=0):
        """One recurrent step.  state: (batch, channels, nstate) float64, updated
        in place; x, delta: (batch, channels); B, C: (batch, nstate).  Returns y."""
        assert state.dtype == np.float64 and state.flags.c_contiguous
        x, delta, A, B, C, D = map(self._f64, (x, delta, A, B, C, D))
        batch, channels, nstate = state.shape
        assert x.shape == (batch, channels) and delta.shape == x.shape
        assert A.shape == (channels, nstate) and B.shape == (batch, nstate) and C.shape == B.shape
        y = np.empty_like(x)
        rc = self._lib.oracle_state_update(self._ptr(state), self._ptr(x), self._ptr(delta),
                                           self._ptr(A), self._ptr(B), self._ptr(C), self._ptr(D),
                                           self._ptr(y), batch, channels, nstate, int(nthreads))
        if rc != 0:
            raise RuntimeError(f"oracle_state_update failed ({rc})")
        return y

    def scan_complex(self, u, delta, A_re, A_im, B, C, D=None, h0=None, want_y=True, nthreads=0):
        """Selective scan with a complex diagonal A = A_re + i A_im and a
        complex state (the Mamba-3 page, "Karmaşık Değerli Durum
        Güncellemesi"; the reading is in ssm_oracle.c).  h0 and the returned
        final state are (batch, channels, nstate, 2) float64, (re, im)
        adjacent.  Returns (y, h_final)."""
        u, delta, A_re, A_im, B, C, D, h0 = map(self._f64, (u, delta, A_re, A_im, B, C, D, h0))
        batch, length, channels = u.shape
        nstate = A_re.shape[1]
        assert delta.shape == u.shape and A_re.shape == (channels, nstate) and A_im.shape == A_re.shape
        assert B.shape == (batch, length, nstate) and C.shape == B.shape
        assert D is None or D.shape == (channels,)
        assert h0 is None or h0.shape == (batch, channels, nstate, 2)
        y = np.empty_like(u) if want_y else None
        hf = np.empty((batch, channels, nstate, 2), dtype=np.float64)
        rc = self._lib.oracle_scan_complex(self._ptr(u), self._ptr(delta), self._ptr(A_re), self._ptr(A_im),
                                           self._ptr(B), self._ptr(C), self._ptr(D), self._ptr(h0), self._ptr(y),
                                           self._ptr(hf), batch, length, channels, nstate, int(nthreads))
        if rc != 0:
            raise RuntimeError(f"oracle_scan_complex failed ({rc})")
        return y, hf

    def scan_mimo(self, u, delta, A, B, C, D=None, h0=None, want_y=True, nthreads=0):
        """Multi-input multi-output scan (the Mamba-3 page, "MIMO Mekanizmasının
        İşleyişi"; the reading is in ssm_oracle.c).  u: (batch, len, ranks,
        channels); delta: (batch, len, channels); B, C: (batch, len, ranks,
        nstate); A: (channels, nstate); D: (channels,) or None; h0: (batch,
        channels, nstate) or None.  Returns (y, h_final), y shaped like u."""
        u, delta, A, B, C, D, h0 = map(self._f64, (u, delta, A, B, C, D, h0))
        batch, length, ranks, channels = u.shape
        nstate = A.shape[1]
        assert delta.shape == (batch, length, channels) and A.shape == (channels, nstate)
        assert B.shape == (batch, length, ranks, nstate) and C.shape == B.shape
        assert D is None or D.shape == (channels,)
        assert h0 is None or h0.shape == (batch, channels, nstate)
        y = np.empty_like(u) if want_y else None
        hf = np.empty((batch, channels, nstate), dtype=np.float64)
        rc = self._lib.oracle_scan_mimo(self._ptr(u), self._ptr(delta), self._ptr(A), self._ptr(B), self._ptr(C),
                                        self._ptr(D), self._ptr(h0), self._ptr(y), self._ptr(hf), batch, length,
                                        channels, nstate, ranks, int(nthreads))
        if rc != 0:
            raise RuntimeError(f"oracle_scan_mimo failed ({rc})")
        return y, hf

    # --- Mamba-2's restricted form (state space duality) -----------------
    @staticmethod
    def _ssd_channel_head(channels: int, headdim: int) -> np.ndarray:
        """Head of every channel: channels are grouped into heads of
        `headdim` consecutive channels, so channel d belongs to head d // headdim."""
        return np.arange(channels) // headdim

    def ssd_scan(self, x, dt, A_head, B, C, D=None, h0=None, headdim=64, want_y=True, nthreads=0, method=0):
        """The scan of Mamba-2's restricted SSM.

        The Mamba-3 page (bitig.info), "Karmaşık Değerli Durum Güncellemesi":
        Mamba-2 reduces the state transition to real scalars; "Mamba SSM
        Nedir? Transformer Alternatifi Rehberi (2026)", "Mamba-2 ve Güncel
        Gelişmeler", and "Albert Gu: Mamba'nın Mucidi ...", "Mamba-2 (2024)":
        under that restriction the SSM equals a masked attention-like form
        (state space duality).  Read plainly: head h has one negative
        scalar a_h, every channel of the head uses A = a_h * I over its
        states, and one step dt[b, t, h] is shared by the head's channels.
        Everything else (discretisation, recurrence, output, skip term) is the
        selective scan's.  So the definition is the scan oracle on inputs
        broadcast to channels: A[d, n] = a_{h(d)}, delta[b, t, d] = dt[b, t, h(d)].

        x: (batch, len, heads*headdim); dt: (batch, len, heads); A_head:
        (heads,); B, C: (batch, len, nstate); D: (channels,) or None; h0:
        (batch, channels, nstate) or None.  Returns (y, h_final) in float64."""
        x, dt, A_head, B = map(self._f64, (x, dt, A_head, B))
        batch, length, channels = x.shape
        heads = A_head.shape[0]
        assert channels == heads * headdim and dt.shape == (batch, length, heads)
        nstate = B.shape[2]
        head_of = self._ssd_channel_head(channels, headdim)
        delta = np.ascontiguousarray(dt[:, :, head_of])
        A = np.ascontiguousarray(np.repeat(A_head[head_of][:, None], nstate, axis=1))
        return self.scan(x, delta, A, B, C, D, h0, want_y=want_y, nthreads=nthreads, method=method)

    def max_threads(self) -> int:
        return int(self._lib.oracle_max_threads())


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from `ssm_oracle.c` (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def scan(*args, **kwargs):
    return get().scan(*args, **kwargs)


def state_update(*args, **kwargs):
    return get().state_update(*args, **kwargs)


def ssd_scan(*args, **kwargs):
    return get().ssd_scan(*args, **kwargs)


def scan_complex(*args, **kwargs):
    return get().scan_complex(*args, **kwargs)


def scan_mimo(*args, **kwargs):
    return get().scan_mimo(*args, **kwargs)

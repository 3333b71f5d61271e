"""Pins for the oracle of Mamba-2's restricted scan (`Oracle.ssd_scan`).

Sources (web pages on the Mamba selective SSM):
  the Mamba-3 page (bitig.info), "Karmaşık Değerli Durum Güncellemesi":
       Mamba-2 reduces the state transition to real scalars;
  "Mamba SSM Nedir? Transformer Alternatifi Rehberi (2026)", "Mamba-2 ve
       Güncel Gelişmeler", and "Albert Gu: Mamba'nın Mucidi ...", "Mamba-2
       (2024)": with that restriction the SSM equals a masked, attention-like
       matrix form (state space duality).

The oracle computes the restricted scan as a recurrence (the scan oracle on
inputs broadcast from heads to channels).  These tests compute the same
outputs by other routes: the dual matrix form (a lower-triangular T x T
matrix per head applied to the head's channels, numpy matmuls), with the
per-token ZOH step taken from van Loan's block matrix exponential; and the
chunked decomposition (intra-chunk matrix form plus chunk-to-chunk states)
that a tensor-core kernel evaluates.
"""
import math

import numpy as np
import pytest
import scipy.linalg

import oracle as oracle_pkg


def _inputs(rng, batch, length, heads, headdim, nstate, with_h0=False):
    x = rng.standard_normal((batch, length, heads * headdim))
    dt = np.exp(rng.uniform(math.log(1e-3), math.log(0.3), (batch, length, heads)))
    A = -np.exp(rng.uniform(0.0, math.log(16.0), heads))
    B = rng.standard_normal((batch, length, nstate))
    C = rng.standard_normal((batch, length, nstate))
    D = rng.standard_normal(heads * headdim)
    h0 = 0.3 * rng.standard_normal((batch, heads * headdim, nstate)) if with_h0 else None
    return x, dt, A, B, C, D, h0


def _step_weights(a, dts, method):
    """Per-token decay and input weight of h' = a h + b x over a step dt:
    zero-order hold from expm([[a dt, dt], [0, 0]]) = [[abar, w], [0, 1]]
    (van Loan), exponential Euler keeps abar and takes w = dt."""
    abar = np.empty_like(dts)
    w = np.empty_like(dts)
    for i, d in enumerate(dts):
        E = scipy.linalg.expm(np.array([[a * d, d], [0.0, 0.0]]))
        abar[i] = E[0, 0]
        w[i] = E[0, 1] if method == 0 else d
    return abar, w


def _dual_form(x, dt, A, B, C, D, h0, headdim, method=0):
    """y = (L o C B^T) (w x) + D x per head, L[t, s] = prod_{s<r<=t} abar_r."""
    batch, length, channels = x.shape
    heads = A.shape[0]
    nstate = B.shape[2]
    y = np.zeros_like(x)
    hf = np.zeros((batch, channels, nstate))
    for b in range(batch):
        G = C[b] @ B[b].T                                   # (T, T): C_t . B_s
        for h in range(heads):
            abar, w = _step_weights(A[h], dt[b, :, h], method)
            logd = np.cumsum(np.log(abar))                   # log prod_{r<=t} abar_r
            Lm = np.tril(np.exp(logd[:, None] - logd[None, :]))
            cols = slice(h * headdim, (h + 1) * headdim)
            X = x[b, :, cols]                                # (T, P)
            y[b, :, cols] = (G * Lm * w[None, :]) @ X
            # state after the last token: sum_s L[T-1, s] w_s B_s x_s^T
            S = (Lm[-1] * w)[:, None] * X                    # (T, P)
            hf[b, cols, :] = S.T @ B[b]
            if h0 is not None:
                H0 = h0[b, cols, :]                          # (P, N)
                y[b, :, cols] += np.exp(logd)[:, None] * (C[b] @ H0.T)
                hf[b, cols, :] += np.exp(logd[-1]) * H0
    if D is not None:
        y += D[None, None, :] * x
    return y, hf


def _chunked(x, dt, A, B, C, D, h0, headdim, chunk, method=0):
    """The chunked evaluation: within a chunk the dual form from a zero state,
    plus the entering state decayed to each token; the state passed to the
    next chunk is the entering one decayed over the chunk plus the chunk's own."""
    batch, length, channels = x.shape
    heads = A.shape[0]
    nstate = B.shape[2]
    y = np.zeros_like(x)
    hf = np.zeros((batch, channels, nstate))
    for b in range(batch):
        for h in range(heads):
            cols = slice(h * headdim, (h + 1) * headdim)
            S = np.zeros((headdim, nstate)) if h0 is None else h0[b, cols, :].copy()
            abar, w = _step_weights(A[h], dt[b, :, h], method)
            for t0 in range(0, length, chunk):
                t1 = min(length, t0 + chunk)
                logd = np.cumsum(np.log(abar[t0:t1]))
                Lm = np.tril(np.exp(logd[:, None] - logd[None, :]))
                X = x[b, t0:t1, cols]
                G = C[b, t0:t1] @ B[b, t0:t1].T
                y[b, t0:t1, cols] = (G * Lm * w[None, t0:t1]) @ X + np.exp(logd)[:, None] * (C[b, t0:t1] @ S.T)
                S = np.exp(logd[-1]) * S + ((Lm[-1] * w[t0:t1])[:, None] * X).T @ B[b, t0:t1]
            hf[b, cols, :] = S
    if D is not None:
        y += D[None, None, :] * x
    return y, hf


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(1e-300, np.max(np.abs(b))))


@pytest.mark.parametrize("method", [0, 1], ids=["zoh", "euler"])
@pytest.mark.parametrize("with_h0", [False, True], ids=["h0=0", "h0"])
def test_ssd_oracle_equals_dual_matrix_form(oracle_lib, method, with_h0):
    rng = np.random.default_rng(4101 + method + 2 * with_h0)
    x, dt, A, B, C, D, h0 = _inputs(rng, 2, 37, 3, 4, 5, with_h0)
    y, hf = oracle_lib.ssd_scan(x, dt, A, B, C, D, h0=h0, headdim=4, method=method)
    yd, hd = _dual_form(x, dt, A, B, C, D, h0, 4, method)
    assert _rel(y, yd) < 1e-11
    assert _rel(hf, hd) < 1e-11


@pytest.mark.parametrize("chunk", [1, 5, 16, 64])
def test_ssd_oracle_equals_chunked_form(oracle_lib, chunk):
    rng = np.random.default_rng(4200 + chunk)
    x, dt, A, B, C, D, h0 = _inputs(rng, 1, 50, 2, 3, 4, with_h0=True)
    y, hf = oracle_lib.ssd_scan(x, dt, A, B, C, D, h0=h0, headdim=3)
    yc, hc = _chunked(x, dt, A, B, C, D, h0, 3, chunk)
    assert _rel(y, yc) < 1e-11
    assert _rel(hf, hc) < 1e-11


def test_ssd_heads_are_independent(oracle_lib):
    """Changing one head's inputs (x block, dt column, a) changes only that
    head's outputs; B and C are shared by all heads."""
    rng = np.random.default_rng(4300)
    x, dt, A, B, C, D, _ = _inputs(rng, 2, 20, 3, 2, 4)
    y1, h1 = oracle_lib.ssd_scan(x, dt, A, B, C, D, headdim=2)
    x2, dt2, A2 = x.copy(), dt.copy(), A.copy()
    x2[:, :, 2:4] = rng.standard_normal(x2[:, :, 2:4].shape)
    dt2[:, :, 1] *= 1.7
    A2[1] *= 0.5
    y2, h2 = oracle_lib.ssd_scan(x2, dt2, A2, B, C, D, headdim=2)
    keep = np.r_[0:2, 4:6]
    assert np.array_equal(y1[:, :, keep], y2[:, :, keep])
    assert np.array_equal(h1[:, keep], h2[:, keep])
    assert _rel(y1[:, :, 2:4], y2[:, :, 2:4]) > 1e-3


@pytest.mark.parametrize("method", [0, 1], ids=["zoh", "euler"])
def test_ssd_one_state_constant_step_closed_form(oracle_lib, method):
    """One head of one channel, one state, constant dt, B = C = 1, x = 1:
    h_t = w (1 - r^(t+1)) / (1 - r) with r = exp(a dt) and the input weight
    w = (r - 1)/a (zero-order hold) or w = dt (exponential Euler)."""
    L, a, d = 30, -2.0, 0.05
    x = np.ones((1, L, 1))
    dt = np.full((1, L, 1), d)
    B = np.ones((1, L, 1))
    C = np.ones((1, L, 1))
    y, hf = oracle_lib.ssd_scan(x, dt, np.array([a]), B, C, None, headdim=1, method=method)
    r = math.exp(a * d)
    w = (r - 1.0) / a if method == 0 else d
    want = np.array([w * (1 - r ** (t + 1)) / (1 - r) for t in range(L)])
    assert np.max(np.abs(y[0, :, 0] - want)) < 1e-14
    assert abs(hf[0, 0, 0] - want[-1]) < 1e-14


def test_ssd_mutant_head_mapping_is_caught(oracle_lib, monkeypatch):
    """Plant a plausible mistake in the oracle (channels dealt to heads
    round-robin instead of in blocks) and check that the dual-form pin fails."""
    rng = np.random.default_rng(4400)
    x, dt, A, B, C, D, _ = _inputs(rng, 1, 24, 3, 4, 4)
    yd, _ = _dual_form(x, dt, A, B, C, D, None, 4)
    monkeypatch.setattr(oracle_pkg.Oracle, "_ssd_channel_head",
                        staticmethod(lambda channels, headdim: np.arange(channels) % (channels // headdim)))
    y, _ = oracle_lib.ssd_scan(x, dt, A, B, C, D, headdim=4)
    assert _rel(y, yd) > 1e-3

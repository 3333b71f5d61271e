"""Pins of the oracle's multi-input multi-output (MIMO) scan, oracle.scan_mimo.

Reading (the Mamba-3 page, bitig.info, "MIMO Mekanizmasının İşleyişi" and
"Seçici Durum Güncellemesindeki İyileştirmeler"; no formula is printed):
per channel, R inputs x^(r) and R outputs y^(r) share one state and one step
Delta; the zero-order hold of "Mamba SSM Nedir? ...", "Ayrık Zamana Geçiş"
with B an N x R matrix,
    h_t = exp(Delta A) h_{t-1} + sum_r (Delta A)^-1 (exp(Delta A) - 1) Delta B^(r) x^(r),
    y_t^(r) = C_t^(r) . h_t + D x_t^(r).

Each pin reaches the result by a route that does not retype the oracle's
formula: the single-input scan (itself pinned in test_oracle_pins.py) at
R = 1 and by superposition, van Loan's block exponential of the whole
multi-input system for the LTI matrix kernel, a hand closed form, linearity
and channel independence.
"""
import math

import numpy as np
import pytest
import scipy.linalg


def _inputs(rng, batch, length, ranks, channels, nstate, dlo=1e-3, dhi=0.5):
    u = rng.standard_normal((batch, length, ranks, channels))
    delta = np.exp(rng.uniform(math.log(dlo), math.log(dhi), (batch, length, channels)))
    A = -np.exp(rng.uniform(math.log(0.1), math.log(10.0), (channels, nstate)))
    B = rng.standard_normal((batch, length, ranks, nstate))
    C = rng.standard_normal((batch, length, ranks, nstate))
    D = rng.standard_normal(channels)
    return u, delta, A, B, C, D


def test_mimo_rank_one_is_the_scan(oracle_lib):
    rng = np.random.default_rng(51)
    u, delta, A, B, C, D = _inputs(rng, 2, 40, 1, 5, 4)
    h0 = rng.standard_normal((2, 5, 4))
    y, hf = oracle_lib.scan_mimo(u, delta, A, B, C, D, h0=h0)
    y1, hf1 = oracle_lib.scan(u[:, :, 0], delta, A, B[:, :, 0], C[:, :, 0], D, h0=h0)
    assert np.array_equal(y[:, :, 0], y1) and np.array_equal(hf, hf1)


@pytest.mark.parametrize("ranks", [2, 3, 8])
def test_mimo_is_a_superposition_of_single_input_scans(oracle_lib, ranks):
    """The recurrence is linear in its input term and Delta does not depend on
    x, so the state is the sum of R single-input scans (input r only), and
    output r reads it with its own C^(r)."""
    rng = np.random.default_rng(52 + ranks)
    u, delta, A, B, C, D = _inputs(rng, 2, 30, ranks, 6, 4)
    h0 = rng.standard_normal((2, 6, 4))
    y, hf = oracle_lib.scan_mimo(u, delta, A, B, C, D, h0=h0)
    h_sum = np.zeros_like(hf)
    y_ref = np.zeros_like(y)
    for rin in range(ranks):
        h_init = h0 if rin == 0 else None
        _, h_r = oracle_lib.scan(u[:, :, rin], delta, A, B[:, :, rin], C[:, :, 0], None, h0=h_init)
        h_sum += h_r
        for rout in range(ranks):
            y_part, _ = oracle_lib.scan(u[:, :, rin], delta, A, B[:, :, rin], C[:, :, rout], None, h0=h_init)
            y_ref[:, :, rout] += y_part
    y_ref += D[None, None, None, :] * u
    np.testing.assert_allclose(hf, h_sum, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12)


def test_mimo_lti_matrix_kernel(oracle_lib):
    """Constant Delta, B, C: y^(r)_t = sum_r' sum_k K^(r,r')_k x^(r')_{t-k} + D x^(r)_t
    with K^(r,r')_k = C^(r) Abar^k Bbar^(r'), Abar and the N x R Bbar from van
    Loan's block exponential expm(Delta [[A, B], [0, 0]]) of the whole system."""
    rng = np.random.default_rng(53)
    L, R, N, dt = 24, 3, 4, 0.09
    a = -np.array([0.3, 1.0, 2.5, 7.0])
    Bm = rng.standard_normal((N, R))
    Cm = rng.standard_normal((R, N))
    M = np.zeros((N + R, N + R))
    M[:N, :N] = np.diag(a)
    M[:N, N:] = Bm
    E = scipy.linalg.expm(dt * M)
    Abar, Bbar = E[:N, :N], E[:N, N:]
    x = rng.standard_normal((L, R))
    K = [Cm @ np.linalg.matrix_power(Abar, k) @ Bbar for k in range(L)]     # (R, R) each
    D = 0.4
    ref = np.array([sum(K[k] @ x[t - k] for k in range(t + 1)) + D * x[t] for t in range(L)])
    u = x.reshape(1, L, R, 1)
    delta = np.full((1, L, 1), dt)
    B = np.broadcast_to(Bm.T, (1, L, R, N)).copy()
    C = np.broadcast_to(Cm, (1, L, R, N)).copy()
    y, _ = oracle_lib.scan_mimo(u, delta, a.reshape(1, N), B, C, np.array([D]))
    np.testing.assert_allclose(y[0, :, :, 0], ref, rtol=1e-11, atol=1e-12)


def test_mimo_hand_closed_form(oracle_lib):
    """One state, A = -ln 2, Delta = 1: Abar = 1/2 and Bbar^(r) = B^(r) / (2 ln 2).
    An impulse on input 1 only, with B^(1) = 2 ln 2, puts h_0 = 1 and then
    h_t = 2^-t; input 0 carries B^(0) = 5 but x^(0) = 0.  Output 0 reads with
    C^(0) = 1, output 1 with C^(1) = 3, and D = 0.5 adds 0.5 to y^(1)_0."""
    L = 6
    u = np.zeros((1, L, 2, 1))
    u[0, 0, 1, 0] = 1.0
    delta = np.ones((1, L, 1))
    A = np.array([[-math.log(2.0)]])
    B = np.zeros((1, L, 2, 1))
    B[0, :, 0, 0] = 5.0
    B[0, :, 1, 0] = 2.0 * math.log(2.0)
    C = np.zeros((1, L, 2, 1))
    C[0, :, 0, 0] = 1.0
    C[0, :, 1, 0] = 3.0
    y, hf = oracle_lib.scan_mimo(u, delta, A, B, C, np.array([0.5]))
    h = 2.0 ** -np.arange(L)
    np.testing.assert_allclose(y[0, :, 0, 0], h, rtol=1e-14)
    want1 = 3.0 * h
    want1[0] += 0.5
    np.testing.assert_allclose(y[0, :, 1, 0], want1, rtol=1e-14)
    np.testing.assert_allclose(hf[0, 0], [2.0 ** -(L - 1)], rtol=1e-14)


def test_mimo_linear_in_x_and_channels_independent(oracle_lib):
    rng = np.random.default_rng(54)
    u, delta, A, B, C, D = _inputs(rng, 2, 20, 4, 7, 8)
    u2 = rng.standard_normal(u.shape)
    y1, _ = oracle_lib.scan_mimo(u, delta, A, B, C, None)
    y2, _ = oracle_lib.scan_mimo(u2, delta, A, B, C, None)
    y12, _ = oracle_lib.scan_mimo(2.0 * u - 0.5 * u2, delta, A, B, C, None)
    np.testing.assert_allclose(y12, 2.0 * y1 - 0.5 * y2, rtol=1e-10, atol=1e-12)
    # permuting channels permutes the outputs and final states (no channel mixing; layout)
    perm = rng.permutation(7)
    y, hf = oracle_lib.scan_mimo(u, delta, A, B, C, D)
    yp, hfp = oracle_lib.scan_mimo(u[..., perm], delta[..., perm], A[perm], B, C, D[perm])
    assert np.array_equal(yp, y[..., perm]) and np.array_equal(hfp, hf[:, perm])


def test_mimo_empty_sequence(oracle_lib):
    A = -np.ones((3, 4))
    h0 = np.arange(2 * 3 * 4, dtype=np.float64).reshape(2, 3, 4)
    z = np.zeros((2, 0, 2, 3))
    y, hf = oracle_lib.scan_mimo(z, np.zeros((2, 0, 3)), A, np.zeros((2, 0, 2, 4)), np.zeros((2, 0, 2, 4)),
                                 None, h0=h0)
    assert y.shape == (2, 0, 2, 3) and np.array_equal(hf, h0)

"""Pins for the fp64 oracle: facts that the pages and the mathematics fix,
checked by routes that do not reuse the oracle's own formulas.

Sources (web pages on the Mamba selective SSM):
  P5 = "Mamba SSM Nedir? Transformer Alternatifi Rehberi (2026)":
       "State Space Model Temelleri" (continuous system with D x),
       "Ayrık Zamana Geçiş" (ZOH discretisation, recurrence, recurrent <-> convolution
       equivalence), "Mamba'nın Yeniliği: Selective SSM" (per-token B, C, Delta),
       "Paralel Tarama Algoritması" (parallel prefix scan).
  P1 = "Mamba: Transformer'a Meydan Okuyan Uzun-Bağımlı Model" (S4 as convolution).

Independent routes used here: van Loan's block matrix exponential for the
exact ZOH step (scipy.linalg.expm), a numerical ODE solve of the continuous
system (scipy.integrate.solve_ivp), direct and FFT convolution (numpy), hand
closed forms in tests/golden/, and algebraic invariants.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_inputs(rng, batch, length, channels, nstate, dlo=1e-3, dhi=1e-1):
    u = rng.standard_normal((batch, length, channels))
    delta = np.exp(rng.uniform(math.log(dlo), math.log(dhi), (batch, length, channels)))
    A = -np.exp(rng.uniform(math.log(0.1), math.log(20.0), (channels, nstate)))
    B = rng.standard_normal((batch, length, nstate))
    C = rng.standard_normal((batch, length, nstate))
    D = rng.standard_normal(channels)
    return u, delta, A, B, C, D


def _zoh_van_loan(a_diag, b_vec, dt):
    """Exact ZOH step of h' = A h + B x via expm([[A, B], [0, 0]] dt) =
    [[Abar, Bbar], [0, 1]] (van Loan, 1978) -- no closed form for Bbar used."""
    n = len(a_diag)
    M = np.zeros((n + 1, n + 1))
    M[:n, :n] = np.diag(a_diag) * dt
    M[:n, n] = b_vec * dt
    E = scipy.linalg.expm(M)
    return np.diag(E[:n, :n]).copy(), E[:n, n].copy()


# --- pin: hand-derived closed forms (golden fixtures) -------------------------

def test_golden_halving_step_response(oracle_lib):
    g = json.load(open(os.path.join(GOLDEN, "zoh_halving_step_response.json")))
    L = len(g["y"])
    u = np.full((1, L, 1), g["x"])
    delta = np.full((1, L, 1), g["delta"])
    A = np.array([[g["A"]]])
    B = np.full((1, L, 1), g["B"])
    C = np.full((1, L, 1), g["C"])
    D = np.array([g["D"]])
    y, hf = oracle_lib.scan(u, delta, A, B, C, D)
    np.testing.assert_allclose(y[0, :, 0], g["y"], rtol=1e-14, atol=1e-15)
    assert hf[0, 0, 0] == pytest.approx(g["h"][-1], rel=1e-14)


def test_golden_impulse_two_states(oracle_lib):
    g = json.load(open(os.path.join(GOLDEN, "zoh_impulse_two_states.json")))
    L = len(g["x"])
    u = np.array(g["x"]).reshape(1, L, 1)
    delta = np.full((1, L, 1), g["delta"])
    A = np.array([g["A"]])
    B = np.tile(np.array(g["B"]), (1, L, 1))
    C = np.tile(np.array(g["C"]), (1, L, 1))
    D = np.array([g["D"]])
    y, _ = oracle_lib.scan(u, delta, A, B, C, D)
    np.testing.assert_allclose(y[0, :, 0], g["y"], rtol=1e-14)


# --- pin: ZOH step equals the exact continuous solution -----------------------

def test_zoh_step_matches_van_loan_and_ode(oracle_lib):
    """P5 'Ayrık Zamana Geçiş': ZOH holds x_t constant over a step of length
    Delta_t.  One oracle step from a non-zero state must equal the exact
    solution of h' = A h + B x, computed two independent ways."""
    rng = np.random.default_rng(1)
    N = 5
    A = -np.exp(rng.uniform(-2, 2.5, (1, N)))
    h0 = rng.standard_normal((1, 1, N))
    for dt in (1e-6, 3e-3, 0.37, 4.0):
        x = rng.standard_normal()
        Bt = rng.standard_normal(N)
        u = np.array([[[x]]])
        delta = np.array([[[dt]]])
        _, hf = oracle_lib.scan(u, delta, A, Bt.reshape(1, 1, N), np.zeros((1, 1, N)), None, h0=h0)
        ab, bb = _zoh_van_loan(A[0], Bt, dt)
        np.testing.assert_allclose(hf[0, 0], ab * h0[0, 0] + bb * x, rtol=1e-11, atol=1e-15)
        sol = scipy.integrate.solve_ivp(lambda _t, h: A[0] * h + Bt * x, (0.0, dt), h0[0, 0],
                                        method="DOP853", rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(hf[0, 0], sol.y[:, -1], rtol=1e-9, atol=1e-13)


def test_selective_sequence_matches_piecewise_ode(oracle_lib):
    """The whole selective recurrence (Delta_t, B_t, C_t varying per token,
    P5 'Selective SSM') equals integrating the continuous system token by
    token with that token's parameters, and y_t = C_t h_t + D x_t reads the
    state after the update at t."""
    rng = np.random.default_rng(2)
    L, Dch, N = 12, 2, 3
    u, delta, A, B, C, D = _rand_inputs(rng, 1, L, Dch, N, 1e-2, 1.0)
    y, hf = oracle_lib.scan(u, delta, A, B, C, D)
    for d in range(Dch):
        h = np.zeros(N)
        for t in range(L):
            x, dt = u[0, t, d], delta[0, t, d]
            sol = scipy.integrate.solve_ivp(lambda _t, hh: A[d] * hh + B[0, t] * x, (0.0, dt), h,
                                            method="DOP853", rtol=1e-12, atol=1e-15)
            h = sol.y[:, -1]
            assert y[0, t, d] == pytest.approx(C[0, t] @ h + D[d] * x, rel=1e-8, abs=1e-12)
        np.testing.assert_allclose(hf[0, d], h, rtol=1e-8, atol=1e-12)


# --- pin: recurrent mode == convolution mode in the LTI case ------------------

def _lti_inputs(rng, L, N, dt):
    A = -np.exp(rng.uniform(-1.5, 1.5, (1, N)))
    Bv = rng.standard_normal(N)
    Cv = rng.standard_normal(N)
    u = rng.standard_normal((1, L, 1))
    delta = np.full((1, L, 1), dt)
    B = np.tile(Bv, (1, L, 1))
    C = np.tile(Cv, (1, L, 1))
    return u, delta, A, B, C, Bv, Cv


def test_lti_equals_direct_convolution(oracle_lib):
    """P5 'Ayrık Zamana Geçiş' (and P1 on S4): with Delta, B, C constant the
    recurrence equals y = K * x + D x with K_k = C Abar^k Bbar."""
    rng = np.random.default_rng(3)
    L, N = 64, 4
    u, delta, A, B, C, Bv, Cv = _lti_inputs(rng, L, N, 0.05)
    D = np.array([0.7])
    y, _ = oracle_lib.scan(u, delta, A, B, C, D)
    ab, bb = _zoh_van_loan(A[0], Bv, 0.05)
    K = np.array([(Cv * ab ** k * bb).sum() for k in range(L)])
    x = u[0, :, 0]
    ref = np.array([sum(K[k] * x[t - k] for k in range(t + 1)) for t in range(L)]) + 0.7 * x
    np.testing.assert_allclose(y[0, :, 0], ref, rtol=1e-11, atol=1e-13)


def test_lti_equals_fft_convolution_long(oracle_lib):
    rng = np.random.default_rng(4)
    L, N = 4096, 16
    u, delta, A, B, C, Bv, Cv = _lti_inputs(rng, L, N, 0.01)
    y, _ = oracle_lib.scan(u, delta, A, B, C, None)
    ab, bb = _zoh_van_loan(A[0], Bv, 0.01)
    k = np.arange(L)
    K = (Cv[None, :] * ab[None, :] ** k[:, None] * bb[None, :]).sum(axis=1)
    n = 2 * L
    ref = np.fft.irfft(np.fft.rfft(K, n) * np.fft.rfft(u[0, :, 0], n), n)[:L]
    scale = np.abs(ref).max()
    assert np.abs(y[0, :, 0] - ref).max() <= 1e-11 * scale


# --- pin: limits of the discretisation ----------------------------------------

def test_delta_to_zero_gives_skip_only(oracle_lib):
    """Delta -> 0: Abar -> 1, Bbar -> 0, so from h = 0 the output is D x,
    with a deviation of order Delta."""
    rng = np.random.default_rng(5)
    u, _, A, B, C, D = _rand_inputs(rng, 2, 50, 3, 4)
    for dt in (1e-14, 1e-10):
        delta = np.full(u.shape, dt)
        y, hf = oracle_lib.scan(u, delta, A, B, C, D)
        dev = np.abs(y - D[None, None, :] * u).max()
        assert dev <= 1e4 * dt                # O(Delta): sum over 50 tokens of |Delta B x| |C|
        assert dev > 0.0                      # the state path is not simply dropped
        assert np.abs(hf).max() <= 1e3 * dt


def test_delta_to_infinity_is_memoryless(oracle_lib):
    """Delta -> inf with A < 0: Abar -> 0 and Bbar -> -B/A, so
    y_t = sum_n C_t[n] (-B_t[n] / A_n) x_t + D x_t with no memory."""
    rng = np.random.default_rng(6)
    u, _, A, B, C, D = _rand_inputs(rng, 2, 20, 3, 4)
    A = -np.abs(A) - 0.5
    delta = np.full(u.shape, 1e4)
    y, _ = oracle_lib.scan(u, delta, A, B, C, D)
    ref = np.einsum("btn,dn,btn->btd", C, -1.0 / A, B) * u + D[None, None, :] * u
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12)


# --- pin: brute-force unrolled sum --------------------------------------------

def test_unrolled_sum_bruteforce(oracle_lib):
    """h_t = sum_{s<=t} (prod_{r=s+1..t} Abar_r) Bbar_s x_s, the recurrence
    written out, with each step's (Abar, Bbar) from van Loan's exponential."""
    rng = np.random.default_rng(7)
    bsz, L, Dch, N = 2, 17, 3, 4
    u, delta, A, B, C, D = _rand_inputs(rng, bsz, L, Dch, N, 1e-2, 2.0)
    y, hf = oracle_lib.scan(u, delta, A, B, C, D)
    for b in range(bsz):
        for d in range(Dch):
            steps = [_zoh_van_loan(A[d], B[b, t], delta[b, t, d]) for t in range(L)]
            for t in range(L):
                h = np.zeros(N)
                for s in range(t + 1):
                    w = np.ones(N)
                    for r in range(s + 1, t + 1):
                        w = w * steps[r][0]
                    h = h + w * steps[s][1] * u[b, s, d]
                assert y[b, t, d] == pytest.approx(C[b, t] @ h + D[d] * u[b, t, d], rel=1e-10, abs=1e-13)
            np.testing.assert_allclose(hf[b, d], h, rtol=1e-10, atol=1e-14)


# --- pin: scan == chain of single-token updates ------------------------------

def test_scan_equals_decode_chain(oracle_lib):
    """The recurrent (generation) mode applied token by token reproduces the
    scan exactly: same state, same outputs (bit for bit in fp64)."""
    rng = np.random.default_rng(8)
    bsz, L, Dch, N = 3, 40, 5, 16
    u, delta, A, B, C, D = _rand_inputs(rng, bsz, L, Dch, N)
    h0 = 0.1 * rng.standard_normal((bsz, Dch, N))
    y, hf = oracle_lib.scan(u, delta, A, B, C, D, h0=h0)
    state = h0.copy()
    for t in range(L):
        yt = oracle_lib.state_update(state, u[:, t], delta[:, t], A, B[:, t], C[:, t], D)
        assert np.array_equal(yt, y[:, t])
    assert np.array_equal(state, hf)


# --- pin: chunk stitching with the linear-recurrence monoid -------------------

def test_chunk_stitch_monoid(oracle_lib):
    """P5 'Paralel Tarama Algoritması' names a parallel prefix scan.  With the
    operator (P1, H1) o (P2, H2) = (P2 P1, P2 H1 + H2) over chunk aggregates
    (P = exp(A * sum of Delta over the chunk), H = chunk-end state from zero)
    any split of the sequence gives the sequential final state."""
    rng = np.random.default_rng(9)
    bsz, L, Dch, N = 2, 300, 3, 8
    u, delta, A, B, C, D = _rand_inputs(rng, bsz, L, Dch, N)
    _, h_full = oracle_lib.scan(u, delta, A, B, C, D)
    for cuts in ([0, 1, 300], [0, 100, 200, 300], [0, 7, 8, 150, 299, 300], [0, 300]):
        P = np.ones((bsz, Dch, N))
        H = np.zeros((bsz, Dch, N))
        for a, b in zip(cuts[:-1], cuts[1:]):
            _, Hk = oracle_lib.scan(u[:, a:b], delta[:, a:b], A, B[:, a:b], C[:, a:b], D)
            Pk = np.exp(A[None] * delta[:, a:b].sum(axis=1)[..., None])
            P, H = Pk * P, Pk * H + Hk
        np.testing.assert_allclose(H, h_full, rtol=1e-12, atol=1e-15)


def test_initial_state_enters_linearly(oracle_lib):
    """h_0 != 0 adds exactly prod(Abar) h_0 to the state and
    sum_n C_t[n] P_t[n] h_0[n] to the outputs (linearity of the recurrence)."""
    rng = np.random.default_rng(10)
    bsz, L, Dch, N = 1, 30, 2, 6
    u, delta, A, B, C, D = _rand_inputs(rng, bsz, L, Dch, N)
    h0 = rng.standard_normal((bsz, Dch, N))
    y1, hf1 = oracle_lib.scan(u, delta, A, B, C, D, h0=h0)
    y0, hf0 = oracle_lib.scan(u, delta, A, B, C, D)
    S = np.cumsum(delta, axis=1)                                  # (b, L, d)
    P = np.exp(S[..., None] * A[None, None])                      # (b, L, d, n)
    np.testing.assert_allclose(hf1 - hf0, P[:, -1] * h0, rtol=1e-11, atol=1e-14)
    corr = np.einsum("btn,btdn,bdn->btd", C, P, h0)
    np.testing.assert_allclose(y1 - y0, corr, rtol=1e-10, atol=1e-13)


# --- pin: linearity in x ------------------------------------------------------

def test_linearity_in_x(oracle_lib):
    rng = np.random.default_rng(11)
    u1, delta, A, B, C, D = _rand_inputs(rng, 2, 64, 4, 16)
    u2 = rng.standard_normal(u1.shape)
    a, b = 0.75, -1.25
    y1, h1 = oracle_lib.scan(u1, delta, A, B, C, D)
    y2, h2 = oracle_lib.scan(u2, delta, A, B, C, D)
    y3, h3 = oracle_lib.scan(a * u1 + b * u2, delta, A, B, C, D)
    np.testing.assert_allclose(y3, a * y1 + b * y2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(h3, a * h1 + b * h2, rtol=1e-11, atol=1e-12)


# --- structure: channels independent, B/C shared, layout by index -------------

def test_layout_and_channel_independence(oracle_lib):
    """Each (batch, channel) row only sees its own u/Delta column, its own row
    of A and D, and its batch's B_t, C_t; the state layout is
    [batch][channel][state]."""
    rng = np.random.default_rng(12)
    bsz, L, Dch, N = 3, 25, 4, 5
    u, delta, A, B, C, D = _rand_inputs(rng, bsz, L, Dch, N)
    y, hf = oracle_lib.scan(u, delta, A, B, C, D)
    for b in range(bsz):
        for d in range(Dch):
            ys, hs = oracle_lib.scan(u[b:b + 1, :, d:d + 1], delta[b:b + 1, :, d:d + 1], A[d:d + 1],
                                     B[b:b + 1], C[b:b + 1], D[d:d + 1])
            assert np.array_equal(ys[0, :, 0], y[b, :, d])
            assert np.array_equal(hs[0, 0], hf[b, d])


def test_empty_sequence(oracle_lib):
    u = np.zeros((2, 0, 3))
    _, hf = oracle_lib.scan(u, u, -np.ones((3, 4)), np.zeros((2, 0, 4)), np.zeros((2, 0, 4)), None)
    assert hf.shape == (2, 3, 4) and not hf.any()


# --- discretisations named on the Mamba-3 page -----------------------------------------
# "Geliştirilmiş Ayrıklaştırma Şeması": Mamba-1/2 used the Euler method, Mamba-3 the
# trapezoidal rule.  Readings (ssm_oracle.c): exponential Euler keeps exp(Delta A) and
# takes Bbar = Delta B; the trapezoid rule takes the step's input integral from the
# previous token (weighted by exp(Delta A)) and the current one, Delta/2 each.

def _impulse_inputs(L, delta, a, b, c):
    x = np.zeros((1, L, 1))
    x[0, 0, 0] = 1.0
    x[0, 7, 0] = -0.5                                   # a second impulse: superposition
    return (x, np.full((1, L, 1), delta), np.array([a]), np.tile(np.array(b), (1, L, 1)),
            np.tile(np.array(c), (1, L, 1)))


@pytest.mark.parametrize("method", ["euler", "trapezoid"])
def test_methods_impulse_response_closed_form(oracle_lib, method):
    """Constant Delta, B, C: the response to an impulse at t=0 is, in closed form,
    exponential Euler  h_k = Abar^k Delta B          (k >= 0)
    trapezoid          h_0 = Delta/2 B,  h_k = Abar^k Delta B  (k >= 1)
    (the previous-token term of step 1 carries the other half, decayed once);
    a second impulse adds its shifted, scaled copy."""
    L, dt = 20, 0.3
    a, b, c = [-0.5, -2.0, -7.0], [1.0, -0.4, 0.25], [0.3, 1.1, -0.8]
    u, delta, A, B, C = _impulse_inputs(L, dt, a, b, c)
    m = oracle_lib.EULER if method == "euler" else oracle_lib.TRAPEZOID
    y, _ = oracle_lib.scan(u, delta, A, B, C, None, method=m)
    abar = np.exp(dt * np.array(a))
    k = np.arange(L)[:, None]
    resp = (abar[None, :] ** k) * dt * np.array(b)[None, :]        # Abar^k Delta B
    if method == "trapezoid":
        resp[0] = 0.5 * dt * np.array(b)
    kernel = resp @ np.array(c)                                      # C . h_k
    expect = kernel.copy()
    expect[7:] += -0.5 * kernel[:L - 7]
    np.testing.assert_allclose(y[0, :, 0], expect, rtol=1e-13, atol=1e-15)


def test_methods_order_of_accuracy(oracle_lib):
    """Against the continuous system h' = A h + B x(t) with a smooth input that
    starts at x(0) = 0 (solved by scipy to 1e-12): zero-order hold and exponential
    Euler converge at first order in Delta, the trapezoidal rule at second order."""
    a = np.array([-1.0, -3.0])
    b = np.array([1.0, 0.5])
    c = np.array([1.0, 1.0])
    T = 4.0

    def xf(t):
        return np.sin(2.0 * t) + 0.5 * np.sin(0.7 * t)

    def exact(ts):
        sol = scipy.integrate.solve_ivp(lambda t, h: a * h + b * xf(t), (0.0, T), [0.0, 0.0],
                                        t_eval=ts, rtol=1e-12, atol=1e-14, method="DOP853")
        return c @ sol.y

    errs = {}
    for dt in (0.02, 0.01):
        L = int(round(T / dt))
        ts = dt * np.arange(1, L + 1)            # token t closes the step ending at (t+1) Delta
        ref = exact(ts)
        u = xf(ts).reshape(1, L, 1)
        delta = np.full((1, L, 1), dt)
        B = np.tile(b, (1, L, 1))
        C = np.tile(c, (1, L, 1))
        for name, m in (("zoh", oracle_lib.ZOH), ("euler", oracle_lib.EULER), ("trap", oracle_lib.TRAPEZOID)):
            y, _ = oracle_lib.scan(u, delta, a[None, :], B, C, None, method=m)
            errs[(name, dt)] = np.max(np.abs(y[0, :, 0] - ref))
    for name, lo, hi in (("zoh", 1.6, 2.4), ("euler", 1.6, 2.4), ("trap", 3.3, 4.7)):
        ratio = errs[(name, 0.02)] / errs[(name, 0.01)]
        assert lo < ratio < hi, f"{name}: error ratio {ratio:.2f} for halved Delta"
    assert errs[("trap", 0.01)] < 0.1 * errs[("euler", 0.01)]


@pytest.mark.parametrize("method", ["euler", "trapezoid"])
def test_methods_share_the_zoh_transition(oracle_lib, method):
    """All three discretisations keep Abar = exp(Delta A), so the part of y that an
    initial state contributes (y(h0) - y(0), linear in h0) is the same as under
    zero-order hold; and as Delta -> 0 the output tends to D x."""
    rng = np.random.default_rng(11)
    u, delta, A, B, C, D = _rand_inputs(rng, 2, 30, 3, 4)
    h0 = rng.standard_normal((2, 3, 4))
    m = oracle_lib.EULER if method == "euler" else oracle_lib.TRAPEZOID
    y1, _ = oracle_lib.scan(u, delta, A, B, C, D, h0=h0, method=m)
    y0, _ = oracle_lib.scan(u, delta, A, B, C, D, method=m)
    z1, _ = oracle_lib.scan(u, delta, A, B, C, D, h0=h0)
    z0, _ = oracle_lib.scan(u, delta, A, B, C, D)
    np.testing.assert_allclose(y1 - y0, z1 - z0, rtol=1e-10, atol=1e-12)
    tiny = np.full_like(delta, 1e-14)
    yt, _ = oracle_lib.scan(u, tiny, A, B, C, D, method=m)
    np.testing.assert_allclose(yt, u * D[None, None, :], rtol=0, atol=1e-12)


# --- backward of the zero-order-hold scan -------------------------------------------------
# Reverse mode of the same recurrence (training).  Pinned by finite differences of the
# forward oracle (itself pinned above), by the LTI closed form of du (a correlation with the
# convolution kernel), and by linearity in the upstream gradient.

def _loss(oracle_lib, args, dy, dh):
    u, delta, A, B, C, D, h0 = args
    y, hf = oracle_lib.scan(u, delta, A, B, C, D, h0=h0)
    return float((y * dy).sum() + (hf * dh).sum())


def test_backward_matches_finite_differences(oracle_lib):
    rng = np.random.default_rng(21)
    u, delta, A, B, C, D = _rand_inputs(rng, 2, 5, 3, 4, dlo=0.05, dhi=0.5)
    h0 = rng.standard_normal((2, 3, 4))
    dy = rng.standard_normal(u.shape)
    dh = rng.standard_normal(h0.shape)
    g = oracle_lib.scan_backward(u, delta, A, B, C, D, dy, h0=h0, dh_final=dh)
    args = [u, delta, A, B, C, D, h0]
    names = ["du", "ddelta", "dA", "dB", "dC", "dD", "dh0"]
    for i, name in enumerate(names):
        base = args[i]
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            step = 1e-6 * max(1.0, abs(base[idx]))
            plus, minus = base.copy(), base.copy()
            plus[idx] += step
            minus[idx] -= step
            a_p, a_m = list(args), list(args)
            a_p[i], a_m[i] = plus, minus
            fd[idx] = (_loss(oracle_lib, a_p, dy, dh) - _loss(oracle_lib, a_m, dy, dh)) / (2 * step)
        np.testing.assert_allclose(g[name], fd, rtol=2e-6, atol=1e-8, err_msg=name)


def _dbbar_da_series(dt, a, terms=40):
    """d/dA of (exp(dt A) - 1)/A from the power series of exp, term by term:
    (e^{dt A} - 1)/A = sum_{k>=1} dt^k A^{k-1}/k!, so its derivative is
    sum_{k>=2} (k-1) dt^k A^{k-2}/k!.  No closed form, no psi()."""
    total, fact = 0.0, 1.0
    for k in range(1, terms + 1):
        fact *= k
        if k >= 2:
            total += (k - 1) * dt ** k * a ** (k - 2) / fact
    return total


@pytest.mark.parametrize("dt, a", [(1e-3, -1e-3), (1e-3, -0.1), (1e-3, -0.9), (1e-3, -5.0), (0.05, -1.0)])
def test_backward_da_small_z(oracle_lib, dt, a):
    """One token from h = 0: dA comes from d Bbar / dA alone, at |Delta A| from
    1e-6 to 5e-2, on both sides of the oracle's switch to a series for small
    |z|.  Reference: the power series of exp differentiated term by term."""
    rng = np.random.default_rng(24)
    N = 3
    u = np.array([[[0.7]]])
    delta = np.array([[[dt]]])
    A = np.full((1, N), a) * np.array([[1.0, 1.5, 2.0]])
    B = rng.standard_normal((1, 1, N))
    C = rng.standard_normal((1, 1, N))
    dy = np.array([[[1.3]]])
    g = oracle_lib.scan_backward(u, delta, A, B, C, np.zeros(1), dy)
    ref = np.array([1.3 * C[0, 0, n] * B[0, 0, n] * 0.7 * _dbbar_da_series(dt, A[0, n]) for n in range(N)])
    np.testing.assert_allclose(g["dA"][0], ref, rtol=1e-12, atol=0)


def test_backward_lti_du_is_correlation_with_kernel(oracle_lib):
    """Constant Delta, B, C: y = K * x + D x, so du_t = sum_k K_k dy_{t+k} + D dy_t."""
    rng = np.random.default_rng(22)
    L, N = 48, 4
    u, delta, A, B, C, Bv, Cv = _lti_inputs(rng, L, N, 0.07)
    D = np.array([0.3])
    dy = rng.standard_normal(u.shape)
    g = oracle_lib.scan_backward(u, delta, A, B, C, D, dy)
    ab, bb = _zoh_van_loan(A[0], Bv, 0.07)
    K = np.array([(Cv * ab ** k * bb).sum() for k in range(L)])
    ref = np.array([sum(K[k] * dy[0, t + k, 0] for k in range(L - t)) for t in range(L)]) + 0.3 * dy[0, :, 0]
    np.testing.assert_allclose(g["du"][0, :, 0], ref, rtol=1e-10, atol=1e-12)


def test_backward_linear_in_upstream_gradient(oracle_lib):
    rng = np.random.default_rng(23)
    u, delta, A, B, C, D = _rand_inputs(rng, 2, 9, 3, 4)
    d1, d2 = rng.standard_normal(u.shape), rng.standard_normal(u.shape)
    g1 = oracle_lib.scan_backward(u, delta, A, B, C, D, d1)
    g2 = oracle_lib.scan_backward(u, delta, A, B, C, D, d2)
    g12 = oracle_lib.scan_backward(u, delta, A, B, C, D, 2.0 * d1 - d2)
    for k in ("du", "ddelta", "dA", "dB", "dC", "dD", "dh0"):
        np.testing.assert_allclose(g12[k], 2.0 * g1[k] - g2[k], rtol=1e-10, atol=1e-12, err_msg=k)

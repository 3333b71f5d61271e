"""Pins for the oracle of the complex-valued state (`Oracle.scan_complex`).

Source: the Mamba-3 page (bitig.info), "Karmaşık Değerli Durum
Güncellemesi" (complex state update; complex eigenvalues represent rotation
and oscillation).  The page gives no formula; the reading (diagonal complex
A, the zero-order hold of "Mamba SSM Nedir? Transformer Alternatifi Rehberi
(2026)", "Ayrık Zamana Geçiş", in complex arithmetic, real B and C, y from the
real part of the state) is stated in oracle/ssm_oracle.c.

Independent routes: a complex state h = p + i q with A = a + i w is the real
two-dimensional system (p, q)' = [[a, -w], [w, a]] (p, q) + (B, 0) x, whose
exact zero-order-hold step is van Loan's block exponential (scipy expm of a
3 x 3 real matrix, no complex arithmetic); the real scan oracle (already
pinned) for w = 0; direct convolution for constant parameters; and symmetry.
"""
import math

import numpy as np
import scipy.linalg


def _inputs(rng, batch, length, channels, nstate):
    u = rng.standard_normal((batch, length, channels))
    delta = np.exp(rng.uniform(math.log(1e-3), math.log(0.3), (batch, length, channels)))
    A_re = -np.exp(rng.uniform(math.log(0.1), math.log(10.0), (channels, nstate)))
    A_im = rng.uniform(-8.0, 8.0, (channels, nstate))
    B = rng.standard_normal((batch, length, nstate))
    C = rng.standard_normal((batch, length, nstate))
    D = rng.standard_normal(channels)
    return u, delta, A_re, A_im, B, C, D


def _real_block_step(a, w, b, dt):
    """Exact ZOH step of the real 2-D system: returns (Abar 2x2, Bbar 2)."""
    M = np.zeros((3, 3))
    M[:2, :2] = np.array([[a, -w], [w, a]]) * dt
    M[0, 2] = b * dt
    E = scipy.linalg.expm(M)
    return E[:2, :2], E[:2, 2]


def _real_block_scan(u, delta, A_re, A_im, B, C, D, h0=None):
    """The recurrence in real 2-D blocks, token by token."""
    batch, length, channels = u.shape
    nstate = A_re.shape[1]
    y = np.zeros_like(u)
    hf = np.zeros((batch, channels, nstate, 2))
    for b in range(batch):
        for d in range(channels):
            h = np.zeros((nstate, 2)) if h0 is None else h0[b, d].copy()
            for t in range(length):
                acc = 0.0
                for n in range(nstate):
                    Ab, Bb = _real_block_step(A_re[d, n], A_im[d, n], B[b, t, n], delta[b, t, d])
                    h[n] = Ab @ h[n] + Bb * u[b, t, d]
                    acc += C[b, t, n] * h[n, 0]
                y[b, t, d] = acc + (D[d] * u[b, t, d] if D is not None else 0.0)
            hf[b, d] = h
    return y, hf


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(1e-300, np.max(np.abs(b))))


def test_complex_reduces_to_real_scan(oracle_lib):
    rng = np.random.default_rng(5101)
    u, delta, A_re, _, B, C, D = _inputs(rng, 2, 40, 3, 4)
    y, hf = oracle_lib.scan_complex(u, delta, A_re, np.zeros_like(A_re), B, C, D)
    yr, hr = oracle_lib.scan(u, delta, A_re, B, C, D)
    assert _rel(y, yr) < 1e-13
    assert _rel(hf[..., 0], hr) < 1e-13
    assert np.max(np.abs(hf[..., 1])) == 0.0


def test_complex_equals_exact_real_block_recurrence(oracle_lib):
    rng = np.random.default_rng(5102)
    u, delta, A_re, A_im, B, C, D = _inputs(rng, 2, 25, 2, 3)
    h0 = 0.5 * rng.standard_normal((2, 2, 3, 2))
    y, hf = oracle_lib.scan_complex(u, delta, A_re, A_im, B, C, D, h0=h0)
    yb, hb = _real_block_scan(u, delta, A_re, A_im, B, C, D, h0=h0)
    assert _rel(y, yb) < 1e-11
    assert _rel(hf, hb) < 1e-11


def test_complex_lti_convolution(oracle_lib):
    """Constant step, B and C: y_t = sum_k K_k x_{t-k} + D x_t with the kernel
    K_k = sum_n C_n [Abar_n^k Bbar_n]_re from the real block step."""
    rng = np.random.default_rng(5103)
    L, N = 48, 3
    u = rng.standard_normal((1, L, 1))
    dt = 0.07
    A_re = -np.array([[0.5, 2.0, 7.0]])
    A_im = np.array([[3.0, -1.5, 12.0]])
    Bv = rng.standard_normal(N)
    Cv = rng.standard_normal(N)
    D = np.array([0.3])
    y, _ = oracle_lib.scan_complex(u, np.full((1, L, 1), dt), A_re, A_im, np.tile(Bv, (1, L, 1)),
                                   np.tile(Cv, (1, L, 1)), D)
    K = np.zeros(L)
    for n in range(N):
        Ab, Bb = _real_block_step(A_re[0, n], A_im[0, n], Bv[n], dt)
        v = Bb.copy()
        for k in range(L):
            K[k] += Cv[n] * v[0]
            v = Ab @ v
    x = u[0, :, 0]
    want = np.array([sum(K[k] * x[t - k] for k in range(t + 1)) for t in range(L)]) + D[0] * x
    assert _rel(y[0, :, 0], want) < 1e-11


def test_complex_conjugate_symmetry(oracle_lib):
    """With real B, C and x, turning every rotation the other way conjugates
    the state and leaves y unchanged."""
    rng = np.random.default_rng(5104)
    u, delta, A_re, A_im, B, C, D = _inputs(rng, 1, 30, 2, 4)
    y1, h1 = oracle_lib.scan_complex(u, delta, A_re, A_im, B, C, D)
    y2, h2 = oracle_lib.scan_complex(u, delta, A_re, -A_im, B, C, D)
    assert _rel(y2, y1) < 1e-12
    assert _rel(h2[..., 0], h1[..., 0]) < 1e-12
    assert _rel(h2[..., 1], -h1[..., 1]) < 1e-12


def test_complex_initial_state_response(oracle_lib):
    """x = 0: only the initial state (re, im adjacent) is carried, turned and
    decayed by the real block steps."""
    rng = np.random.default_rng(5105)
    u, delta, A_re, A_im, B, C, _ = _inputs(rng, 1, 20, 2, 3)
    u[:] = 0.0
    h0 = rng.standard_normal((1, 2, 3, 2))
    y, hf = oracle_lib.scan_complex(u, delta, A_re, A_im, B, C, None, h0=h0)
    yb, hb = _real_block_scan(u, delta, A_re, A_im, B, C, None, h0=h0)
    assert _rel(y, yb) < 1e-11
    assert _rel(hf, hb) < 1e-11


def test_complex_quarter_turn_halving_closed_form(oracle_lib):
    """Delta = 1, A = -ln 2 + i pi/2: exp(Delta A) = i/2 exactly (half a
    magnitude, a quarter turn per step).  With B = C = 1 and an impulse
    x_0 = 1, h_t = (i/2)^t Bbar with Bbar = (i/2 - 1) / A; in real arithmetic
    (a + ib)/(c + id) = ((ac + bd) + i(bc - ad)) / (c^2 + d^2), so
    Re Bbar = (ln 2 + pi/4) / (ln^2 2 + pi^2/4), Im Bbar = (pi/2 - ln 2 / 2) / (same).
    Then y_0 = Re Bbar, y_1 = -Im Bbar / 2, y_{t+2} = -y_t / 4, and after six
    tokens h_5 = (i/32) Bbar = (-Im Bbar / 32, Re Bbar / 32)."""
    L = 6
    ln2, hp = math.log(2.0), math.pi / 2
    den = ln2 * ln2 + hp * hp
    re_b, im_b = (ln2 + math.pi / 4) / den, (hp - ln2 / 2) / den
    u = np.zeros((1, L, 1))
    u[0, 0, 0] = 1.0
    y, hf = oracle_lib.scan_complex(u, np.ones((1, L, 1)), np.array([[-ln2]]), np.array([[hp]]),
                                    np.ones((1, L, 1)), np.ones((1, L, 1)), None)
    want = [re_b, -im_b / 2]
    for t in range(2, L):
        want.append(-want[t - 2] / 4)
    assert np.max(np.abs(y[0, :, 0] - np.array(want))) < 1e-14
    assert abs(hf[0, 0, 0, 0] - (-im_b / 32)) < 1e-15 and abs(hf[0, 0, 0, 1] - re_b / 32) < 1e-15

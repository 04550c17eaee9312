"""Pins of the fp64 oracle against what the Mamba-3 pages fix (CPU only).

Each test checks the oracle against something other than itself: a special
case that reduces to a textbook recurrence, an independently written route
through the same equations, a closed form, a hand-computed fixture, or an
invariant of the mathematics.
"""
import math

import numpy as np
import pytest

import oracle
import routes
from conftest import read_golden

RNG_TOL = 1e-11


def rand_inputs(rng, b, T, H, G, P, N, R, theta_max=1.0, with_state=True):
    x = rng.standard_normal((b, T, H, R, P))
    B = rng.standard_normal((b, T, G, R, N)) / math.sqrt(N)
    C = rng.standard_normal((b, T, G, R, N)) / math.sqrt(N)
    dt = np.log1p(np.exp(rng.standard_normal((b, T, H)) - 1.0))
    A = -np.exp(0.5 * rng.standard_normal((b, T, H)))
    lam = 1.0 / (1.0 + np.exp(-rng.standard_normal((b, T, H))))
    theta = rng.uniform(-theta_max, theta_max, (b, T, G, N // 2))
    D = rng.standard_normal(H)
    st = {}
    if with_state:
        st = dict(h0=rng.standard_normal((b, H, N, P)),
                  x_prev=rng.standard_normal((b, H, R, P)),
                  B_prev=rng.standard_normal((b, G, R, N)) / math.sqrt(N))
    return dict(x=x, B=B, C=C, dt=dt, A=A, lam=lam, theta=theta, D=D), st


def rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# --- special cases ----------------------------------------------------------------

@pytest.mark.parametrize("R", [1, 3])
def test_euler_reduction(R):
    """lam = 1, theta = 0 gives exponential-Euler (Mamba-2), Remark 2."""
    rng = np.random.default_rng(1)
    inp, st = rand_inputs(rng, 2, 40, 4, 2, 5, 6, R)
    inp["lam"][:] = 1.0
    inp["theta"][:] = 0.0
    y, hT, _, _ = oracle.scan(**inp, **st)
    ye, he = routes.euler_loop(inp["x"], inp["B"], inp["C"], inp["dt"], inp["A"], inp["D"],
                               h0=st["h0"])
    assert rel(y, ye) < RNG_TOL and rel(hT, he) < RNG_TOL


def test_euler_reduction_drops_previous_token():
    """With lam = 1 the beta term vanishes, so the carried previous token is irrelevant."""
    rng = np.random.default_rng(2)
    inp, st = rand_inputs(rng, 1, 10, 2, 1, 3, 4, 2)
    inp["lam"][:] = 1.0
    y1, h1, _, _ = oracle.scan(**inp, **st)
    st2 = dict(st, x_prev=st["x_prev"] * 0.0, B_prev=st["B_prev"] * 0.0)
    y2, h2, _, _ = oracle.scan(**inp, **st2)
    assert np.array_equal(y1, y2) and np.array_equal(h1, h2)


def test_theta_zero_gives_real_state():
    """theta = 0 with zero imaginary inputs keeps the imaginary state slots exactly 0
    ("The Expressivity Bottleneck": a real transition only scales the state)."""
    rng = np.random.default_rng(3)
    inp, st = rand_inputs(rng, 1, 30, 2, 1, 4, 8, 2)
    inp["theta"][:] = 0.0
    inp["B"][..., 1::2] = 0.0
    st["h0"][:, :, 1::2, :] = 0.0
    st["B_prev"][..., 1::2] = 0.0
    y, hT, _, _ = oracle.scan(**inp, **st)
    assert np.all(hT[:, :, 1::2, :] == 0.0)
    assert np.any(hT[:, :, 0::2, :] != 0.0)
    # then C's imaginary slots cannot influence y
    inp2 = dict(inp)
    inp2["C"] = inp["C"].copy()
    inp2["C"][..., 1::2] = 123.0
    y2, _, _, _ = oracle.scan(**inp2, **st)
    assert np.array_equal(y, y2)


# --- independent routes -------------------------------------------------------------

@pytest.mark.parametrize("R,G", [(1, 1), (2, 2), (3, 1)])
def test_bruteforce_txt(R, G):
    """Materialised Y = (L o C~B~^T) X with L = L_decay . L_band, fresh sequence."""
    rng = np.random.default_rng(10 + R)
    inp, _ = rand_inputs(rng, 2, 24, 2, G, 3, 6, R, with_state=False)
    y, _, _, _ = oracle.scan(**inp)
    yb = routes.bruteforce_txt(**inp)
    assert rel(y, yb) < RNG_TOL


@pytest.mark.parametrize("angle", [False, True])
def test_complex_route(angle):
    """Complex-valued SSM with exp(dt (A + i theta)) transition (Propositions 2, 4)."""
    rng = np.random.default_rng(20)
    inp, st = rand_inputs(rng, 2, 33, 3, 3, 4, 8, 2, theta_max=3.0)
    y, hT, xp, bp = oracle.scan(**inp, **st, theta_is_angle=angle)
    yc, hc = routes.complex_route(**inp, **st, theta_is_angle=angle)
    assert rel(y, yc) < RNG_TOL and rel(hT, hc) < RNG_TOL
    assert np.array_equal(xp, inp["x"][:, -1]) and np.array_equal(bp, inp["B"][:, -1])


def test_rope_route():
    """Proposition 4 in the rotated frame, h_T rotated back by the net angle."""
    rng = np.random.default_rng(21)
    inp, st = rand_inputs(rng, 1, 40, 4, 2, 5, 10, 3, theta_max=math.pi)
    y, hT, _, _ = oracle.scan(**inp, **st)
    yr, hr = routes.rope_route(**inp, **st)
    assert rel(y, yr) < 1e-10 and rel(hT, hr) < 1e-10


def test_implicit_convolution_route():
    """Remark 4: trapezoid = width-2 convolution on B x before the Euler recurrence."""
    rng = np.random.default_rng(22)
    inp, st = rand_inputs(rng, 1, 25, 2, 1, 3, 4, 2)
    inp["theta"][:] = 0.0
    y, hT, _, _ = oracle.scan(**inp, **st)
    kw = {k: inp[k] for k in ("x", "B", "C", "dt", "A", "lam", "D")}
    yi, hi = routes.implicit_conv_route(**kw, **st)
    assert rel(y, yi) < RNG_TOL and rel(hT, hi) < RNG_TOL


def test_mimo_is_sum_of_r2_siso():
    """MIMO = R^2 SISO SSMs: H = sum_j h^(j), y^(i) = C^(i)T H
    ("Expressing MIMO as Multiple SISO SSMs")."""
    rng = np.random.default_rng(30)
    R = 3
    inp, st = rand_inputs(rng, 1, 20, 2, 1, 4, 6, R)
    y, hT, _, _ = oracle.scan(**inp, **st)
    ysum = np.zeros_like(y)
    hsum = np.zeros_like(hT)
    for j in range(R):
        for i in range(R):
            sub = dict(inp)
            sub["x"] = inp["x"][:, :, :, j:j + 1]
            sub["B"] = inp["B"][:, :, :, j:j + 1]
            sub["C"] = inp["C"][:, :, :, i:i + 1]
            sub["D"] = None
            h0 = st["h0"] if j == 0 else np.zeros_like(st["h0"])
            yj, hj, _, _ = oracle.scan(**sub, h0=h0, x_prev=st["x_prev"][:, :, j:j + 1],
                                       B_prev=st["B_prev"][:, :, j:j + 1])
            ysum[:, :, :, i] += yj[:, :, :, 0]
            if i == 0:
                hsum += hj
    ysum += inp["D"][None, None, :, None, None] * inp["x"]
    assert rel(y, ysum) < RNG_TOL and rel(hT, hsum) < RNG_TOL


# --- closed forms and worked examples ---------------------------------------------

def _scalar_case(T, dt, A, lam, theta, B, C, x, h0=None, D=None):
    """N = 2 (one pair), P = 1, R = 1, one head; per-token scalars broadcast."""
    f = lambda v: np.broadcast_to(np.asarray(v, dtype=float), (T,)).reshape(1, T, 1)
    Bv = np.broadcast_to(np.asarray(B, float), (T, 2)).reshape(1, T, 1, 1, 2)
    Cv = np.broadcast_to(np.asarray(C, float), (T, 2)).reshape(1, T, 1, 1, 2)
    xv = np.broadcast_to(np.asarray(x, float), (T,)).reshape(1, T, 1, 1, 1)
    th = np.broadcast_to(np.asarray(theta, float), (T,)).reshape(1, T, 1, 1)
    h0a = None if h0 is None else np.asarray(h0, float).reshape(1, 1, 2, 1)
    return oracle.scan(xv, Bv, Cv, f(dt), f(A), f(lam), th, D=D, h0=h0a)


def test_constant_coefficient_closed_form():
    """Constant alpha, beta, gamma, B = x = 1: h_t = h* + alpha^t (gamma - h*),
    h* = (beta + gamma) / (1 - alpha) (unrolled Proposition 1, fresh start)."""
    T, dt, A, lam = 50, 0.7, -0.4, 0.3
    y, hT, _, _ = _scalar_case(T, dt, A, lam, 0.0, [1.0, 0.0], [1.0, 0.0], 1.0)
    al = math.exp(dt * A)
    be, ga = (1 - lam) * dt * al, lam * dt
    hs = (be + ga) / (1 - al)
    t = np.arange(T)
    expect = hs + al ** t * (ga - hs)
    assert np.max(np.abs(y[0, :, 0, 0, 0] - expect)) < 1e-13


def test_damped_rotation_closed_form():
    """B = 0, h0 = (1, 0), C = (0, 1): y_t = alpha^(t+1) sin((t+1) dt theta)
    (the complex eigenvalue A + i theta gives a damped rotation)."""
    T, dt, A, th = 60, 0.3, -0.2, 1.1
    y, _, _, _ = _scalar_case(T, dt, A, 0.5, th, [0.0, 0.0], [0.0, 1.0], 1.0, h0=[1.0, 0.0])
    t = np.arange(1, T + 1)
    expect = np.exp(dt * A) ** t * np.sin(t * dt * th)
    assert np.max(np.abs(y[0, :, 0, 0, 0] - expect)) < 1e-13


def test_parity_worked_example():
    """h_t = R(pi x_t) h_{t-1} computes parity; fixture tests/golden/parity_example.txt."""
    g = read_golden("parity_example.txt")
    bits = np.array(g["bits"])
    T = len(bits)
    y, _, _, _ = _scalar_case(T, 1.0, 0.0, 0.5, math.pi * bits, [0.0, 0.0], [1.0, 0.0], 0.0,
                              h0=[1.0, 0.0])
    assert np.max(np.abs(y[0, :, 0, 0, 0] - np.array(g["expected"]))) < 1e-12


def test_ssd_mask_fixture():
    """Columns of L = L_decay . L_band from the hand-computed T = 3 fixture."""
    g = read_golden("ssd_mask_T3.txt")
    dt, lam, alpha = map(np.array, (g["dt"], g["lam"], g["alpha"]))
    A = np.log(alpha) / dt
    L = np.array(g["L"])
    T = len(dt)
    for s in range(T):
        x = np.zeros(T)
        x[s] = 1.0
        y, _, _, _ = _scalar_case(T, dt, A, lam, 0.0, [1.0, 0.0], [1.0, 0.0], x)
        assert np.max(np.abs(y[0, :, 0, 0, 0] - L[:, s])) < 1e-14


@pytest.mark.parametrize("lam,order", [(0.5, 2.0), (1.0, 1.0)])
def test_convergence_order(lam, order):
    """lam = 1/2 is the trapezoid rule (second order, global error O(dt^2));
    lam = 1 is Euler (first order).  LTI h' = a h + b sin(w tau), exact solution
    from the variation-of-constants formula (Proposition 5)."""
    a, b, w, tend = -1.0, 1.0, 3.0, 2.0
    errs = []
    for dt in (0.02, 0.01, 0.005):
        T = int(round(tend / dt)) + 1
        tau = np.arange(T) * dt
        y, _, _, _ = _scalar_case(T, dt, a, lam, 0.0, [b, 0.0], [1.0, 0.0], np.sin(w * tau))
        errs.append(abs(y[0, -1, 0, 0, 0] - routes.lti_exact(a, b, w, tau[-1])))
    rates = [math.log2(errs[i] / errs[i + 1]) for i in range(2)]
    assert all(abs(r - order) < 0.15 for r in rates), (errs, rates)


# --- invariants --------------------------------------------------------------------

def test_pair_permutation_invariance():
    """Rotations act on disjoint pairs and commute (Proposition 3): relabelling
    the pairs consistently permutes h and leaves y unchanged."""
    rng = np.random.default_rng(40)
    N = 10
    inp, st = rand_inputs(rng, 1, 30, 2, 1, 3, N, 2, theta_max=2.0)
    perm = rng.permutation(N // 2)
    rows = np.stack([2 * perm, 2 * perm + 1], axis=1).reshape(-1)
    inp2 = dict(inp, B=inp["B"][..., rows], C=inp["C"][..., rows],
                theta=inp["theta"][..., perm])
    st2 = dict(st, h0=st["h0"][:, :, rows], B_prev=st["B_prev"][..., rows])
    y, hT, _, _ = oracle.scan(**inp, **st)
    y2, h2, _, _ = oracle.scan(**inp2, **st2)
    assert rel(y2, y) < 1e-14 and rel(h2, hT[:, :, rows]) < 1e-14


def test_call_split_carries_previous_token():
    """Splitting the sequence into two calls and carrying (h, x_prev, B_prev) gives
    the one-call result; dropping the carried token breaks it (beta_0 needs it)."""
    rng = np.random.default_rng(41)
    inp, st = rand_inputs(rng, 2, 50, 2, 1, 3, 6, 2, theta_max=2.0)
    y, hT, xp, bp = oracle.scan(**inp, **st)
    cut = 17
    first = {k: (v[:, :cut] if k not in ("D",) else v) for k, v in inp.items()}
    second = {k: (v[:, cut:] if k not in ("D",) else v) for k, v in inp.items()}
    y1, h1, xp1, bp1 = oracle.scan(**first, **st)
    y2, h2, xp2, bp2 = oracle.scan(**second, h0=h1, x_prev=xp1, B_prev=bp1)
    assert rel(np.concatenate([y1, y2], axis=1), y) < 1e-13 and rel(h2, hT) < 1e-13
    assert np.array_equal(xp2, xp) and np.array_equal(bp2, bp)
    y3, _, _, _ = oracle.scan(**second, h0=h1)
    assert rel(y3[:, :2], y[:, cut:cut + 2]) > 1e-6


def test_decode_steps_equal_scan():
    """T single-token decode steps reproduce the T-token scan."""
    rng = np.random.default_rng(42)
    inp, st = rand_inputs(rng, 2, 12, 2, 2, 3, 4, 2)
    y, hT, _, _ = oracle.scan(**inp, **st)
    h, xp, bp = st["h0"], st["x_prev"], st["B_prev"]
    for t in range(12):
        one = [inp[k][:, t] for k in ("x", "B", "C", "dt", "A", "lam", "theta")]
        yt, h, xp, bp = oracle.decode_step(*one, inp["D"], h, xp, bp)
        assert rel(yt, y[:, t]) < 1e-13
    assert rel(h, hT) < 1e-13


def test_rejects_bad_shapes():
    rng = np.random.default_rng(43)
    inp, _ = rand_inputs(rng, 1, 4, 3, 2, 2, 4, 1)     # H = 3 not divisible by G = 2
    with pytest.raises(ValueError):
        oracle.scan(**inp)

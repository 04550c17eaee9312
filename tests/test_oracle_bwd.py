"""Pins of the oracle's backward pass (reverse-mode gradients of the recurrence) against
central finite differences of the pinned forward oracle.

The pages describe only the forward computation; the backward is its derivative, so the
check is the derivative's definition: for a scalar loss L = <y, Wy> + <h_T, Wh> with random
weights, dL/dv for every element v of every input (x, B, C, dt, A, lam, theta, D and the
initial state h0, x_prev, B_prev) must match (L(v + e) - L(v - e)) / 2e to the central
difference's error (O(e^2) truncation plus rounding), at shapes where each finite difference
is cheap.  Groups shared by two heads (G = 1, H = 2) check the head sums of the B, C and theta
gradients; the pre-scaled angle flag checks the theta path without dt.  Two more, independent
derivations (tests/routes.py) must agree with the oracle's reverse pass through the
recurrence: the hand-derived gradients of the materialised T x T form (fresh sequence), and
the chunked backward with an adjoint state between chunks (any starting state).  Planted
mistakes in a copy of the backward's C source are caught.
"""
import math
import os
import subprocess

import numpy as np
import pytest

import oracle
import routes

SRC = os.path.join(os.path.dirname(oracle.__file__), "m3_oracle.c")
KEYS = ("x", "B", "C", "dt", "A", "lam", "theta", "D", "h0", "x_prev", "B_prev")
GRAD = {"x": "dx", "B": "dB", "C": "dC", "dt": "ddt", "A": "dA", "lam": "dlam",
        "theta": "dtheta", "D": "dD", "h0": "dh0", "x_prev": "dx_prev", "B_prev": "dB_prev"}


def _problem(seed, b=2, T=5, H=2, G=1, P=3, N=4, R=2):
    rng = np.random.default_rng(seed)
    v = dict(
        x=rng.standard_normal((b, T, H, R, P)),
        B=rng.standard_normal((b, T, G, R, N)) / math.sqrt(N),
        C=rng.standard_normal((b, T, G, R, N)) / math.sqrt(N),
        dt=np.log1p(np.exp(rng.standard_normal((b, T, H)) - 1.0)),
        A=-np.exp(0.5 * rng.standard_normal((b, T, H))),
        lam=1.0 / (1.0 + np.exp(-rng.standard_normal((b, T, H)))),
        theta=rng.uniform(-2.0, 2.0, (b, T, G, N // 2)),
        D=rng.standard_normal(H),
        h0=rng.standard_normal((b, H, N, P)),
        x_prev=rng.standard_normal((b, H, R, P)),
        B_prev=rng.standard_normal((b, G, R, N)) / math.sqrt(N),
    )
    Wy = rng.standard_normal((b, T, H, R, P))
    Wh = rng.standard_normal((b, H, N, P))
    return v, Wy, Wh


def _loss(v, Wy, Wh, angle):
    y, hT, _, _ = oracle.scan(v["x"], v["B"], v["C"], v["dt"], v["A"], v["lam"], v["theta"],
                              D=v["D"], h0=v["h0"], x_prev=v["x_prev"], B_prev=v["B_prev"],
                              theta_is_angle=angle, nthreads=1)
    return float(np.sum(y * Wy) + np.sum(hT * Wh))


def _max_fd_error(seed, angle, lib_path=None, **shape):
    """max over inputs of max |analytic - finite difference| / max |finite difference|."""
    v, Wy, Wh = _problem(seed, **shape)
    g = oracle.scan_bwd(v["x"], v["B"], v["C"], v["dt"], v["A"], v["lam"], v["theta"], Wy,
                        D=v["D"], h0=v["h0"], x_prev=v["x_prev"], B_prev=v["B_prev"], dhT=Wh,
                        theta_is_angle=angle, nthreads=1, lib_path=lib_path)
    eps = 1e-6
    worst = 0.0
    for k in KEYS:
        fd = np.zeros_like(v[k])
        flat = v[k].reshape(-1)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + eps
            lp = _loss(v, Wy, Wh, angle)
            flat[i] = keep - eps
            lm = _loss(v, Wy, Wh, angle)
            flat[i] = keep
            fd.reshape(-1)[i] = (lp - lm) / (2 * eps)
        err = np.max(np.abs(g[GRAD[k]] - fd)) / max(np.max(np.abs(fd)), 1e-12)
        worst = max(worst, err)
    return worst


@pytest.mark.parametrize("angle", [False, True])
def test_gradients_match_finite_differences(angle):
    assert _max_fd_error(3 + angle, angle) < 1e-7


def test_gradients_match_finite_differences_rank4():
    """R = 4 (the rank of the MIMO workloads), two groups of one head each."""
    assert _max_fd_error(11, False, b=1, T=5, H=2, G=2, P=3, N=4, R=4) < 1e-7


def test_gradients_match_finite_differences_siso_groups():
    """R = 1, two groups of two heads, odd headdim."""
    assert _max_fd_error(9, False, b=1, T=6, H=4, G=2, P=5, N=6, R=1) < 1e-7


@pytest.mark.parametrize("angle,R,G", [(False, 2, 1), (True, 1, 2), (False, 3, 2)])
def test_gradients_match_materialised_form_derivative(angle, R, G):
    """An independent derivation: the hand-derived gradients of the materialised T x T form
    (L o C~B~^T) X (tests/routes.py) equal the oracle's reverse pass through the recurrence,
    for a fresh sequence."""
    v, Wy, _ = _problem(21 + R, b=2, T=12, H=4, G=G, P=3, N=6, R=R)
    args = [v[k] for k in ("x", "B", "C", "dt", "A", "lam", "theta")]
    g = oracle.scan_bwd(*args, Wy, D=v["D"], theta_is_angle=angle)
    r = routes.bruteforce_bwd(*args, Wy, D=v["D"], theta_is_angle=angle)
    for k in ("dx", "dB", "dC", "ddt", "dA", "dlam", "dtheta", "dD"):
        assert np.max(np.abs(g[k] - r[k])) <= 1e-11 * max(1.0, np.max(np.abs(r[k]))), k


@pytest.mark.parametrize("angle,R,G,chunk,T", [(False, 2, 1, 4, 13), (True, 1, 2, 5, 12),
                                                (False, 3, 2, 3, 10), (False, 1, 1, 16, 9),
                                                (False, 4, 1, 16, 37)])   # 64 (token, rank) rows
def test_gradients_match_chunked_form_derivative(angle, R, G, chunk, T):
    """The chunked backward (adjoint state between chunks in the call's rotated frame,
    materialised-form derivative inside each chunk; tests/routes.py) equals the oracle's
    reverse pass with a starting state, dL/dh_T and ragged chunks."""
    v, Wy, Wh = _problem(31 + R, b=2, T=T, H=4, G=G, P=3, N=6, R=R)
    args = [v[k] for k in ("x", "B", "C", "dt", "A", "lam", "theta")]
    st = dict(D=v["D"], h0=v["h0"], x_prev=v["x_prev"], B_prev=v["B_prev"], dhT=Wh,
              theta_is_angle=angle)
    g = oracle.scan_bwd(*args, Wy, **st)
    r = routes.chunked_bwd(*args, Wy, chunk, **st)
    for k in GRAD.values():
        assert np.max(np.abs(g[k] - r[k])) <= 1e-12 * max(1.0, np.max(np.abs(r[k]))), k


def test_zero_loss_weights_give_zero_gradients():
    v, Wy, Wh = _problem(1)
    g = oracle.scan_bwd(v["x"], v["B"], v["C"], v["dt"], v["A"], v["lam"], v["theta"],
                        np.zeros_like(Wy), D=v["D"], h0=v["h0"], x_prev=v["x_prev"],
                        B_prev=v["B_prev"])
    assert all(np.all(g[k] == 0) for k in g if g[k] is not None)


def test_skip_gradient_closed_form():
    """dL/dD = <dy, x> summed over batch and tokens (Y = h^T C + D x)."""
    v, Wy, Wh = _problem(2)
    g = oracle.scan_bwd(v["x"], v["B"], v["C"], v["dt"], v["A"], v["lam"], v["theta"], Wy,
                        D=v["D"], h0=v["h0"], x_prev=v["x_prev"], B_prev=v["B_prev"], dhT=Wh)
    assert np.allclose(g["dD"], np.einsum("bthrp,bthrp->h", Wy, v["x"]), rtol=1e-13, atol=0)


MUTATIONS = [
    ("adjoint_not_decayed",
     "for (size_t e = 0; e < NP; ++e) Lam[e] = alpha * dM[e];",
     "for (size_t e = 0; e < NP; ++e) Lam[e] = dM[e];"),
    ("rotation_not_transposed",
     "dM[(2 * i) * P + p] = c * l0 + s * l1;",
     "dM[(2 * i) * P + p] = c * l0 - s * l1;"),
    ("beta_path_dropped_for_previous_B",
     "dBp[r * N + n] += beta * v;",
     "dBp[r * N + n] += 0.0 * v;"),
    ("dlam_sign",
     "dlam[bt * H + hh] = -dbeta * dtv * alpha + dgamma * dtv;",
     "dlam[bt * H + hh] = dbeta * dtv * alpha + dgamma * dtv;"),
    ("angle_derivative_uses_h_not_U",
     "const double u0 = ht[(2 * i) * P + p] - gamma * bx0;",
     "const double u0 = ht[(2 * i) * P + p];"),
    ("readout_adjoint_dropped",
     "Lam[n * P + p] += v;",
     "Lam[n * P + p] += 0.0 * v;"),
    ("dt_misses_angle_term",
     "dphi_theta += dphi * th[i];",
     "dphi_theta += 0.0 * th[i];"),
]


def _compile(src_text, out):
    c = out + ".c"
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", out, c,
                           "-lm"])
    return out


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_backward_mutation_is_caught(tmp_path, name, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    lib = _compile(text.replace(old, new), str(tmp_path / f"lib_{name}.so"))
    assert _max_fd_error(4, False, lib_path=lib, b=1, T=4, H=2, G=1, P=2, N=4, R=2) > 1e-4, \
        f"planted mistake '{name}' was not caught"

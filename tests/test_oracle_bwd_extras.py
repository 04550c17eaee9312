"""Pins of the oracle's backward with the fused extras (output gate, BCNorm + BC biases, MIMO
lightweight expansion) against central finite differences of the pinned forward oracle with
the same extras.

For L = <y, Wy> + <h_T, Wh>, every element of every input is checked, including the gate z,
the head biases B_bias / C_bias and the expansion weights x_expand / z_expand.  Separate
cases switch each extra on alone (so a mistake in one chain cannot hide behind another),
then all of them at once with shared groups."""
import math

import numpy as np
import pytest

import oracle


def _problem(seed, gate, bc, xe, ze, b=2, T=4, H=2, G=1, P=3, N=4, R=2):
    rng = np.random.default_rng(seed)
    v = dict(
        x=rng.standard_normal((b, T, H, P) if xe else (b, T, H, R, P)),
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
    if gate:
        v["z"] = rng.standard_normal((b, T, H, P) if ze else (b, T, H, R, P)) * 1.5
    if bc:
        v["B_bias"] = 1.0 + 0.3 * rng.standard_normal((H, N))
        v["C_bias"] = 1.0 + 0.3 * rng.standard_normal((H, N))
    if xe:
        v["x_expand"] = rng.standard_normal((H, R, P))
    if ze:
        v["z_expand"] = rng.standard_normal((H, R, P))
    Wy = rng.standard_normal((b, T, H, R, P))
    Wh = rng.standard_normal((b, H, N, P))
    return v, Wy, Wh, (1e-3 if bc else 0.0)


CORE = ("x", "B", "C", "dt", "A", "lam", "theta")


def _fwd(v, eps):
    kw = {k: v[k] for k in ("D", "h0", "x_prev", "B_prev", "z", "B_bias", "C_bias", "x_expand",
                            "z_expand") if k in v}
    return oracle.scan(*(v[k] for k in CORE), bc_eps=eps, nthreads=1, **kw)


def _max_fd_error(seed, gate, bc, xe, ze, **shape):
    v, Wy, Wh, eps = _problem(seed, gate, bc, xe, ze, **shape)
    kw = {k: v[k] for k in ("D", "h0", "x_prev", "B_prev", "z", "B_bias", "C_bias", "x_expand",
                            "z_expand") if k in v}
    g = oracle.scan_bwd_ex(*(v[k] for k in CORE), Wy, dhT=Wh, bc_eps=eps, nthreads=1, **kw)
    names = {"x": "dx", "B": "dB", "C": "dC", "dt": "ddt", "A": "dA", "lam": "dlam",
             "theta": "dtheta", "D": "dD", "h0": "dh0", "x_prev": "dx_prev", "B_prev": "dB_prev",
             "z": "dz", "B_bias": "dB_bias", "C_bias": "dC_bias", "x_expand": "dx_expand",
             "z_expand": "dz_expand"}

    def loss():
        y, hT, _, _ = _fwd(v, eps)
        return float(np.sum(y * Wy) + np.sum(hT * Wh))

    step = 1e-6
    worst = {}
    for k in v:
        fd = np.zeros_like(v[k])
        flat = v[k].reshape(-1)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + step
            lp = loss()
            flat[i] = keep - step
            lm = loss()
            flat[i] = keep
            fd.reshape(-1)[i] = (lp - lm) / (2 * step)
        worst[k] = float(np.max(np.abs(g[names[k]] - fd)) / max(np.max(np.abs(fd)), 1e-12))
    return worst


@pytest.mark.parametrize("gate,bc,xe,ze", [
    (True, False, False, False),    # output gate alone
    (False, True, False, False),    # BCNorm + biases alone
    (False, False, True, False),    # x expansion alone
    (True, False, False, True),     # gate with z expansion
])
def test_extras_gradients_match_finite_differences(gate, bc, xe, ze):
    worst = _max_fd_error(5, gate, bc, xe, ze)
    assert max(worst.values()) < 1e-7, worst


def test_all_extras_gradients_match_finite_differences_shared_groups():
    worst = _max_fd_error(6, True, True, True, True, b=1, T=4, H=4, G=2, P=2, N=4, R=2)
    assert max(worst.values()) < 1e-7, worst


def test_extras_off_equals_plain_backward():
    """With every extra off the two backward paths agree (up to the order in which the
    group's heads are summed)."""
    v, Wy, Wh, _ = _problem(7, False, False, False, False)
    kw = {k: v[k] for k in ("D", "h0", "x_prev", "B_prev")}
    a = oracle.scan_bwd_ex(*(v[k] for k in CORE), Wy, dhT=Wh, **kw)
    b = oracle.scan_bwd(*(v[k] for k in CORE), Wy, dhT=Wh, **kw)
    for k in b:
        assert np.max(np.abs(a[k] - b[k])) <= 1e-13 * max(1.0, np.max(np.abs(b[k]))), k

"""The oracle pins are strong enough: each plausible mistake, planted in a temporary
copy of the oracle's C source on the CPU, is caught by at least one pin check.

The mutated copy is compiled into pytest's tmp dir and loaded under its own path;
the real oracle library is never touched.
"""
import math
import os
import subprocess

import numpy as np
import pytest

import oracle
import routes

SRC = os.path.join(os.path.dirname(oracle.__file__), "m3_oracle.c")

# (name, exact text in the oracle source, replacement)
MUTATIONS = [
    ("beta_term_not_rotated",
     "h[n * P + p] = alpha * h[n * P + p] + beta * v;",
     "h[n * P + p] = alpha * h[n * P + p]; (void)beta;"),
    ("rotation_sign_flipped",
     "r0[p] = c * m0 - s * m1;\n            r1[p] = s * m0 + c * m1;",
     "r0[p] = c * m0 + s * m1;\n            r1[p] = -s * m0 + c * m1;"),
    ("beta_missing_alpha",
     "const double beta = (1.0 - lam) * dt * alpha;",
     "const double beta = (1.0 - lam) * dt;"),
    ("gamma_uses_one_minus_lam",
     "const double gamma = lam * dt;",
     "const double gamma = (1.0 - lam) * dt;"),
    ("readout_transposed_rank",
     "v += h[n * P + p] * Ct[r * N + n];",
     "v += h[n * P + p] * Ct[((n * 3 + r) % N) + 0 * r];"),
    ("angle_not_scaled_by_dt",
     "const double phi = (flags & M3O_THETA_IS_ANGLE) ? th[i] : dt * th[i];",
     "const double phi = th[i];"),
    ("previous_token_not_carried",
     "memcpy(bp, Bt, sizeof(double) * (size_t)R * N);",
     "(void)Bt;"),
    ("skip_term_dropped",
     "Y[r * P + p] = v + Dh * X[r * P + p];",
     "Y[r * P + p] = v;"),
    ("rank_sum_uses_first_column_only",
     "for (int r = 0; r < R; ++r) v += Bt[r * N + n] * X[r * P + p];",
     "v += Bt[n] * X[p];"),
]


def _inputs(seed, R):
    rng = np.random.default_rng(seed)
    b, T, H, G, P, N = 1, 14, 2, 1, 3, 6
    inp = dict(
        x=rng.standard_normal((b, T, H, R, P)),
        B=rng.standard_normal((b, T, G, R, N)) / math.sqrt(N),
        C=rng.standard_normal((b, T, G, R, N)) / math.sqrt(N),
        dt=np.log1p(np.exp(rng.standard_normal((b, T, H)) - 1.0)),
        A=-np.exp(0.5 * rng.standard_normal((b, T, H))),
        lam=1.0 / (1.0 + np.exp(-rng.standard_normal((b, T, H)))),
        theta=rng.uniform(-2.0, 2.0, (b, T, G, N // 2)),
        D=rng.standard_normal(H),
    )
    st = dict(h0=rng.standard_normal((b, H, N, P)), x_prev=rng.standard_normal((b, H, R, P)),
              B_prev=rng.standard_normal((b, G, R, N)) / math.sqrt(N))
    return inp, st


def _pins_pass(lib_path):
    """A compact subset of the pins: complex route (with carried state), brute-force
    T x T (fresh), both at R = 1 and R = 3."""
    ok = True
    for R in (1, 3):
        inp, st = _inputs(7 + R, R)
        y, hT, _, _ = oracle.scan(**inp, **st, lib_path=lib_path)
        yc, hc = routes.complex_route(**inp, **st)
        ok &= np.max(np.abs(y - yc)) < 1e-10 and np.max(np.abs(hT - hc)) < 1e-10
        yf, _, _, _ = oracle.scan(**inp, lib_path=lib_path)
        ok &= np.max(np.abs(yf - routes.bruteforce_txt(**inp))) < 1e-10
        # carried previous token across a call split
        cut = 5
        first = {k: (v if k == "D" else v[:, :cut]) for k, v in inp.items()}
        second = {k: (v if k == "D" else v[:, cut:]) for k, v in inp.items()}
        _, h1, xp1, bp1 = oracle.scan(**first, **st, lib_path=lib_path)
        y2, _, _, _ = oracle.scan(**second, h0=h1, x_prev=xp1, B_prev=bp1, lib_path=lib_path)
        ok &= np.max(np.abs(y2 - yc[:, cut:])) < 1e-10
    return bool(ok)


def _compile(src_text, out):
    c = out + ".c"
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", out, c,
                           "-lm"])
    return out


def test_unmutated_oracle_passes_the_subset():
    assert _pins_pass(None)


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(tmp_path, name, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    lib = _compile(text.replace(old, new), str(tmp_path / f"lib_{name}.so"))
    assert not _pins_pass(lib), f"planted mistake '{name}' was not caught"

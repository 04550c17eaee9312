"""Pins of the oracle's BC normalisation and BC biases (Mamba-3 paper summary, "Technical
Approach": B and C are RMS-normalised per token after their projection, then a learned
head-specific, channel-wise bias is added).  Each check compares against the plain
oracle (no BC map) or against a property the definition fixes:

  - RMS normalisation is scale invariant: scaling every B and C column (and B_prev) by
    its own positive factor leaves y and h unchanged (epsilon ~ 0);
  - a unit-RMS column is a fixed point: pre-normalised inputs give the plain oracle;
  - with B = C = 0 and G = H, the biases alone act as per-head B and C of the plain
    oracle (the bias is added per head, per state channel, to every rank column);
  - normalise-then-add-bias equals the plain oracle on inputs mapped that way (the
    reverse order fails this).
Planted mistakes in a copy of the oracle source are caught by these checks.
"""
import math
import os
import subprocess

import numpy as np
import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "m3_oracle.c")


def _inputs(seed, R=2, G=3):
    rng = np.random.default_rng(seed)
    b, T, H, P, N = 2, 9, 3, 4, 6
    inp = dict(
        x=rng.standard_normal((b, T, H, R, P)),
        B=rng.standard_normal((b, T, G, R, N)) / math.sqrt(N),
        C=rng.standard_normal((b, T, G, R, N)) / math.sqrt(N),
        dt=np.log1p(np.exp(rng.standard_normal((b, T, H)) - 1.0)),
        A=-np.exp(0.5 * rng.standard_normal((b, T, H))),
        lam=1.0 / (1.0 + np.exp(-rng.standard_normal((b, T, H)))),
        theta=rng.uniform(-1.0, 1.0, (b, T, G, N // 2)),
        D=rng.standard_normal(H),
    )
    st = dict(h0=rng.standard_normal((b, H, N, P)), x_prev=rng.standard_normal((b, H, R, P)),
              B_prev=rng.standard_normal((b, G, R, N)) / math.sqrt(N))
    bias = dict(B_bias=1.0 + 0.3 * rng.standard_normal((H, N)),
                C_bias=1.0 + 0.3 * rng.standard_normal((H, N)))
    return inp, st, bias


def _rms_normalise(v):
    return v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True))


def _close(a, b, tol):
    return np.max(np.abs(a - b)) <= tol * max(1.0, np.max(np.abs(b)))


def _bc_pins_pass(lib_path=None):
    ok = True
    inp, st, bias = _inputs(3)
    eps = 1e-300
    # scale invariance of the normalisation
    rng = np.random.default_rng(9)
    y1, h1, _, _ = oracle.scan(**inp, **st, bc_eps=eps, lib_path=lib_path)
    sc = dict(inp)
    sc["B"] = inp["B"] * rng.uniform(0.2, 5.0, inp["B"].shape[:-1] + (1,))
    sc["C"] = inp["C"] * rng.uniform(0.2, 5.0, inp["C"].shape[:-1] + (1,))
    st2 = dict(st, B_prev=st["B_prev"] * rng.uniform(0.2, 5.0, st["B_prev"].shape[:-1] + (1,)))
    y2, h2, _, _ = oracle.scan(**sc, **st2, bc_eps=eps, lib_path=lib_path)
    ok &= _close(y2, y1, 1e-10) and _close(h2, h1, 1e-10)
    # unit-RMS columns are a fixed point of the normalisation
    un = dict(inp, B=_rms_normalise(inp["B"]), C=_rms_normalise(inp["C"]))
    stn = dict(st, B_prev=_rms_normalise(st["B_prev"]))
    yn, hn, _, _ = oracle.scan(**un, **stn, bc_eps=eps, lib_path=lib_path)
    yp, hp, _, _ = oracle.scan(**un, **stn, lib_path=lib_path)
    ok &= _close(yn, yp, 1e-12) and _close(hn, hp, 1e-12)
    # biases alone act as per-head B and C (G = H, zero data)
    inp3, st3, bias3 = _inputs(4, G=3)
    zb = dict(inp3, B=np.zeros_like(inp3["B"]), C=np.zeros_like(inp3["C"]))
    stz = dict(st3, B_prev=np.zeros_like(st3["B_prev"]))
    yb, hb, _, _ = oracle.scan(**zb, **stz, **bias3, lib_path=lib_path)
    b_, T, H, R = inp3["x"].shape[:4]
    as_data = dict(inp3, B=np.broadcast_to(bias3["B_bias"][None, None, :, None, :],
                                           inp3["B"].shape).copy(),
                   C=np.broadcast_to(bias3["C_bias"][None, None, :, None, :],
                                     inp3["C"].shape).copy())
    std = dict(st3, B_prev=np.broadcast_to(bias3["B_bias"][None, :, None, :],
                                           st3["B_prev"].shape).copy())
    yd, hd, _, _ = oracle.scan(**as_data, **std, lib_path=lib_path)
    ok &= _close(yb, yd, 1e-12) and _close(hb, hd, 1e-12)
    # normalise, then add the bias (G = H so that the mapped B, C are per head)
    eps2 = 1e-6
    ym, hm, _, _ = oracle.scan(**inp3, **st3, **bias3, bc_eps=eps2, lib_path=lib_path)

    def mapped(v, bvec):     # v [..., G=H, R, N], bvec [H, N]
        s = 1.0 / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps2)
        return v * s + bvec[:, None, :]
    mp = dict(inp3, B=mapped(inp3["B"], bias3["B_bias"]), C=mapped(inp3["C"], bias3["C_bias"]))
    stm = dict(st3, B_prev=mapped(st3["B_prev"], bias3["B_bias"]))
    yq, hq, _, _ = oracle.scan(**mp, **stm, lib_path=lib_path)
    ok &= _close(ym, yq, 1e-12) and _close(hm, hq, 1e-12)
    return bool(ok)


def test_bc_pins():
    assert _bc_pins_pass()


def test_bc_map_keeps_raw_B_prev_in_the_state():
    """The state carries the raw previous-token B (the map is applied where it is used)."""
    inp, st, bias = _inputs(6)
    _, _, _, bp = oracle.scan(**inp, **st, **bias, bc_eps=1e-6)
    assert np.array_equal(bp, inp["B"][:, -1])


BC_MUTATIONS = [
    ("eps_outside_sqrt", "scale = 1.0 / sqrt(ss / N + eps);", "scale = 1.0 / sqrt(ss / N) + eps;"),
    ("sum_not_averaged", "scale = 1.0 / sqrt(ss / N + eps);", "scale = 1.0 / sqrt(ss + eps);"),
    ("bias_before_scale",
     "out[r * N + n] = in[r * N + n] * scale + (bias ? bias[n] : 0.0);",
     "out[r * N + n] = (in[r * N + n] + (bias ? bias[n] : 0.0)) * scale;"),
    ("bias_not_added", "out[r * N + n] = in[r * N + n] * scale + (bias ? bias[n] : 0.0);",
     "out[r * N + n] = in[r * N + n] * scale;"),
    ("B_prev_not_mapped",
     "m3o_bc_map(N, R, B_prev + ((size_t)b * G + g) * R * N, bb, bc_eps, bp);",
     "memcpy(bp, B_prev + ((size_t)b * G + g) * R * N, sizeof(double) * (size_t)R * N);"),
]


@pytest.mark.parametrize("name,old,new", BC_MUTATIONS, ids=[m[0] for m in BC_MUTATIONS])
def test_bc_mutation_is_caught(tmp_path, name, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1
    c = tmp_path / f"{name}.c"
    c.write_text(text.replace(old, new))
    lib = str(tmp_path / f"lib_{name}.so")
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", lib,
                           str(c), "-lm"])
    assert not _bc_pins_pass(lib)

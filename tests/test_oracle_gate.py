"""Pins of the oracle's output gate, y <- y * SiLU(z) after the D x skip (Mamba-3 paper
summary, "Technical Approach": output gating multiplies y_t element-wise by SiLU(z_t)).

SiLU(z) = z * sigmoid(z) is pinned by properties the definition fixes, each checked
against the ungated oracle run on the same inputs:
  - z = 0 closes the gate exactly;
  - SiLU(z) - SiLU(-z) = z, so y(z) - y(-z) = y_ungated * z element-wise, with a nonzero
    skip D, so the gate is checked on the readout with the skip included (a sigmoid gate,
    a mirrored SiLU or a plain product fails);
  - the gate saturates: SiLU(40) = 40 to double precision, SiLU(-40) ~ 0.
Planted mistakes in a copy of the gate's C source are caught by these checks.
"""
import math
import os
import subprocess

import numpy as np
import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "m3_oracle.c")


def _inputs(seed, R=2):
    rng = np.random.default_rng(seed)
    b, T, H, G, P, N = 2, 9, 3, 1, 4, 6
    inp = dict(
        x=rng.standard_normal((b, T, H, R, P)),
        B=rng.standard_normal((b, T, G, R, N)) / math.sqrt(N),
        C=rng.standard_normal((b, T, G, R, N)) / math.sqrt(N),
        dt=np.log1p(np.exp(rng.standard_normal((b, T, H)) - 1.0)),
        A=-np.exp(0.5 * rng.standard_normal((b, T, H))),
        lam=1.0 / (1.0 + np.exp(-rng.standard_normal((b, T, H)))),
        theta=rng.uniform(-1.0, 1.0, (b, T, G, N // 2)),
        D=rng.standard_normal(H) + 2.0,
    )
    z = rng.standard_normal((b, T, H, R, P)) * 2.0
    return inp, z


def _gate_pins_pass(lib_path=None):
    inp, z = _inputs(5)
    y0, h0, _, _ = oracle.scan(**inp, lib_path=lib_path)
    ok = True
    yz0, hz0, _, _ = oracle.scan(**inp, z=np.zeros_like(z), lib_path=lib_path)
    ok &= bool(np.all(yz0 == 0.0)) and np.array_equal(hz0, h0)     # gate leaves the state alone
    yp, _, _, _ = oracle.scan(**inp, z=z, lib_path=lib_path)
    ym, _, _, _ = oracle.scan(**inp, z=-z, lib_path=lib_path)
    ok &= np.max(np.abs((yp - ym) - y0 * z)) <= 1e-12 * max(1.0, np.max(np.abs(y0 * z)))
    ys, _, _, _ = oracle.scan(**inp, z=np.full_like(z, 40.0), lib_path=lib_path)
    ok &= np.max(np.abs(ys - 40.0 * y0)) <= 1e-12 * np.max(np.abs(40.0 * y0))
    yn, _, _, _ = oracle.scan(**inp, z=np.full_like(z, -40.0), lib_path=lib_path)
    ok &= np.max(np.abs(yn)) <= 1e-14 * np.max(np.abs(y0))
    return bool(ok)


def test_gate_pins():
    assert _gate_pins_pass()


def test_decode_gate_matches_gated_scan_of_one_token():
    inp, z = _inputs(6)
    one = {k: (v if k == "D" else v[:, :1]) for k, v in inp.items()}
    ys, hs, _, _ = oracle.scan(**one, z=z[:, :1])
    yd, hd, _, _ = oracle.decode_step(*(one[k][:, 0] for k in ("x", "B", "C", "dt", "A", "lam",
                                                                "theta")),
                                      one["D"], np.zeros_like(hs), None, None, z=z[:, 0])
    assert np.array_equal(yd, ys[:, 0]) and np.array_equal(hd, hs)


GATE_MUTATIONS = [
    ("sigmoid_gate", "y[i] *= z[i] / (1.0 + exp(-z[i]));", "y[i] *= 1.0 / (1.0 + exp(-z[i]));"),
    ("mirrored_silu", "y[i] *= z[i] / (1.0 + exp(-z[i]));", "y[i] *= z[i] / (1.0 + exp(z[i]));"),
    ("plain_product", "y[i] *= z[i] / (1.0 + exp(-z[i]));", "y[i] *= z[i];"),
]


@pytest.mark.parametrize("name,old,new", GATE_MUTATIONS, ids=[m[0] for m in GATE_MUTATIONS])
def test_gate_mutation_is_caught(tmp_path, name, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1
    c = tmp_path / f"{name}.c"
    c.write_text(text.replace(old, new))
    lib = str(tmp_path / f"lib_{name}.so")
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", lib,
                           str(c), "-lm"])
    assert not _gate_pins_pass(lib)

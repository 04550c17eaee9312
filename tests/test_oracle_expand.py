"""Pins of the oracle's MIMO lightweight expansion (Mamba-3 paper summary, "Multi-Input,
Multi-Output (MIMO) Formulation", MIMO Parameterization Choices): the per-head input x and
gate z keep P values per token, and a learned data-independent vector w [H][R][P] scales
them element-wise to the P x R MIMO input, X[r][p] = x[p] w[h][r][p].

Each check compares the oracle with something other than itself:
  - a closed form: constant coefficients, B = (1, 0), x = 1 and theta = 0 make every state
    column p an affine scalar recurrence driven by u_p = sum_r w[r][p], unrolled by hand
    (Proposition 1); the readout c_r h_t[p], the skip D w[r][p] and the expanded gate,
    SiLU from torch, follow per (r, p), so a transposed, shared or dropped weight fails;
  - the pages' decomposition of MIMO into R^2 SISO runs ("Expressing MIMO as Multiple SISO
    SSMs"), with SISO input j = x * w[:, j, :];
  - a call split: the expanded previous token carried in the state continues the sequence.
Planted mistakes in a copy of the expansion's C source are caught by these checks.
"""
import math
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "m3_oracle.c")


def _silu(v):
    return torch.nn.functional.silu(torch.as_tensor(v, dtype=torch.float64)).numpy()


def _closed_form_ok(lib_path=None):
    """H = 2 heads with their own weights, R = 3, P = 4, N = 2 (one pair), fresh state."""
    T, H, R, P, N = 40, 2, 3, 4, 2
    dt, A, lam, Dv = 0.6, -0.5, 0.35, 0.7
    rng = np.random.default_rng(5)
    w = rng.uniform(0.2, 1.8, (H, R, P))
    wz = rng.uniform(-1.5, 1.5, (H, R, P))
    cr = np.array([1.0, -0.5, 2.0])
    x = np.ones((1, T, H, P))
    z = rng.standard_normal((1, T, H, P)) * 2.0
    B = np.zeros((1, T, 1, R, N))
    B[..., 0] = 1.0
    C = np.zeros((1, T, 1, R, N))
    C[..., 0] = cr
    f = lambda v: np.full((1, T, H), v)
    kw = dict(dt=f(dt), A=f(A), lam=f(lam), theta=np.zeros((1, T, 1, N // 2)),
              D=np.full(H, Dv), lib_path=lib_path)
    y, hT, xp, _ = oracle.scan(x, B, C, x_expand=w, **kw)
    yg, _, _, _ = oracle.scan(x, B, C, x_expand=w, z=z, z_expand=wz, **kw)

    al = math.exp(dt * A)
    be, ga = (1 - lam) * dt * al, lam * dt
    u = w.sum(axis=1)                                   # [H, P]
    hs = (be + ga) * u / (1 - al)
    t = np.arange(T)[:, None, None]
    h = hs[None] + al ** t * (ga * u[None] - hs[None])  # [T, H, P]
    expect = cr[None, None, :, None] * h[:, :, None, :] + Dv * w[None]   # [T, H, R, P]
    gate = _silu(z[0][:, :, None, :] * wz[None])
    ok = np.max(np.abs(y[0] - expect)) < 1e-12
    ok &= np.max(np.abs(yg[0] - expect * gate)) < 1e-12
    ok &= np.max(np.abs(hT[0, :, 0, :] - h[-1])) < 1e-12 and np.max(np.abs(hT[0, :, 1, :])) == 0
    ok &= np.max(np.abs(xp[0] - w)) == 0                # X_{T-1} = 1 * w
    return bool(ok)


def _decomposition_ok(lib_path=None):
    """Expanded MIMO = sum over input j of the SISO run on x * w[:, j, :] (B column j),
    read out by C column i; no skip (D = None), fresh state."""
    rng = np.random.default_rng(11)
    b, T, H, G, P, N, R = 1, 16, 2, 1, 3, 6, 3
    x = rng.standard_normal((b, T, H, P))
    w = rng.standard_normal((H, R, P))
    inp = dict(
        B=rng.standard_normal((b, T, G, R, N)) / math.sqrt(N),
        C=rng.standard_normal((b, T, G, R, N)) / math.sqrt(N),
        dt=np.log1p(np.exp(rng.standard_normal((b, T, H)) - 1.0)),
        A=-np.exp(0.5 * rng.standard_normal((b, T, H))),
        lam=1.0 / (1.0 + np.exp(-rng.standard_normal((b, T, H)))),
        theta=rng.uniform(-2.0, 2.0, (b, T, G, N // 2)),
    )
    y, _, _, _ = oracle.scan(x, **inp, x_expand=w, lib_path=lib_path)
    ysum = np.zeros_like(y)
    for j in range(R):
        xj = (x * w[None, None, :, j, :])[:, :, :, None, :]
        for i in range(R):
            sub = dict(inp)
            sub["B"] = inp["B"][:, :, :, j:j + 1]
            sub["C"] = inp["C"][:, :, :, i:i + 1]
            yj, _, _, _ = oracle.scan(xj, **sub)
            ysum[:, :, :, i] += yj[:, :, :, 0]
    return bool(np.max(np.abs(y - ysum)) < 1e-11 * max(1.0, np.max(np.abs(ysum))))


def _split_ok(lib_path=None):
    """Two chained expanded calls equal one call: the state carries the expanded X_{T-1}."""
    rng = np.random.default_rng(17)
    b, T, H, G, P, N, R = 2, 12, 2, 1, 4, 6, 2
    x = rng.standard_normal((b, T, H, P))
    w = rng.standard_normal((H, R, P))
    inp = dict(
        B=rng.standard_normal((b, T, G, R, N)) / math.sqrt(N),
        C=rng.standard_normal((b, T, G, R, N)) / math.sqrt(N),
        dt=np.log1p(np.exp(rng.standard_normal((b, T, H)) - 1.0)),
        A=-np.exp(0.5 * rng.standard_normal((b, T, H))),
        lam=1.0 / (1.0 + np.exp(-rng.standard_normal((b, T, H)))),
        theta=rng.uniform(-2.0, 2.0, (b, T, G, N // 2)),
    )
    D = rng.standard_normal(H)
    y, hT, _, _ = oracle.scan(x, **inp, D=D, x_expand=w, lib_path=lib_path)
    cut = 5
    first = {k: v[:, :cut] for k, v in inp.items()}
    second = {k: v[:, cut:] for k, v in inp.items()}
    y1, h1, xp1, bp1 = oracle.scan(x[:, :cut], **first, D=D, x_expand=w, lib_path=lib_path)
    y2, h2, _, _ = oracle.scan(x[:, cut:], **second, D=D, x_expand=w, h0=h1, x_prev=xp1,
                               B_prev=bp1, lib_path=lib_path)
    return bool(np.max(np.abs(np.concatenate([y1, y2], axis=1) - y)) < 1e-12
                and np.max(np.abs(h2 - hT)) < 1e-12)


def test_expansion_closed_form():
    assert _closed_form_ok()


def test_expanded_mimo_is_sum_of_r2_siso():
    assert _decomposition_ok()


def test_expanded_call_split_carries_expanded_token():
    assert _split_ok()


def test_expand_matches_broadcast_definition():
    """The helper's layout: out[..., h, r, p] = v[..., h, p] * w[h, r, p]."""
    rng = np.random.default_rng(3)
    v = rng.standard_normal((2, 5, 3, 4))
    w = rng.standard_normal((3, 2, 4))
    assert np.array_equal(oracle.expand(v, w), v[..., :, None, :] * w)


def test_decode_with_expansion_is_one_token_scan():
    rng = np.random.default_rng(23)
    b, H, G, P, N, R = 2, 2, 1, 4, 6, 4
    x = rng.standard_normal((b, H, P))
    z = rng.standard_normal((b, H, P))
    w, wz = rng.standard_normal((H, R, P)), rng.standard_normal((H, R, P))
    B = rng.standard_normal((b, G, R, N))
    C = rng.standard_normal((b, G, R, N))
    dt, A, lam = rng.uniform(0.1, 1, (b, H)), -rng.uniform(0.1, 1, (b, H)), rng.uniform(0, 1, (b, H))
    th = rng.uniform(-1, 1, (b, G, N // 2))
    D = rng.standard_normal(H)
    h, xp, bp = rng.standard_normal((b, H, N, P)), rng.standard_normal((b, H, R, P)), \
        rng.standard_normal((b, G, R, N))
    yd, hd, xpd, _ = oracle.decode_step(x, B, C, dt, A, lam, th, D, h, xp, bp, z=z,
                                        x_expand=w, z_expand=wz)
    ys, hs, xps, _ = oracle.scan(x[:, None], B[:, None], C[:, None], dt[:, None], A[:, None],
                                 lam[:, None], th[:, None], D=D, h0=h, x_prev=xp, B_prev=bp,
                                 z=z[:, None], x_expand=w, z_expand=wz)
    assert np.array_equal(yd, ys[:, 0]) and np.array_equal(hd, hs) and np.array_equal(xpd, xps)


MUTATIONS = [
    ("weight_index_transposed",
     "in[(i * H + h) * P + p] * w[((size_t)h * R + r) * P + p];",
     "in[(i * H + h) * P + p] * w[((size_t)h * P + p) * R + r];"),
    ("weights_of_head_zero_for_all_heads",
     "in[(i * H + h) * P + p] * w[((size_t)h * R + r) * P + p];",
     "in[(i * H + h) * P + p] * w[((size_t)0 * R + r) * P + p];"),
    ("input_channel_shifted_by_rank",
     "in[(i * H + h) * P + p] * w[((size_t)h * R + r) * P + p];",
     "in[(i * H + h) * P + (p + r) % P] * w[((size_t)h * R + r) * P + p];"),
    ("weight_ignored",
     "in[(i * H + h) * P + p] * w[((size_t)h * R + r) * P + p];",
     "in[(i * H + h) * P + p] + 0.0 * w[((size_t)h * R + r) * P + p];"),
]


def _compile(src_text, out):
    c = out + ".c"
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", out, c,
                           "-lm"])
    return out


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_expansion_mutation_is_caught(tmp_path, name, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    lib = _compile(text.replace(old, new), str(tmp_path / f"lib_{name}.so"))
    caught = not (_closed_form_ok(lib) and _decomposition_ok(lib) and _split_ok(lib))
    assert caught, f"planted mistake '{name}' was not caught"

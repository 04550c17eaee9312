"""Parity of the MIMO lightweight expansion (Mamba-3 paper summary, "Multi-Input,
Multi-Output (MIMO) Formulation", MIMO Parameterization Choices: x and z hold P values per
head, scaled element-wise to P x R by a data-independent [H][R][P] vector) on every kernel,
through the C ABI, against the fp64 oracle on the same rounded inputs.

Besides the oracle comparison, the expanded call must equal, bit for bit, the plain call
given the expanded tensors the library's rounding defines (bf16(x * w) in fp32): the
kernels expand on chip exactly what an expanded io-dtype x would hold."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import KEYS, f64, rel_slices
from state_space_model_06_b200 import inputs, m3

pytestmark = pytest.mark.gpu


def _host_expand(v, w, io):
    """[.., H, P] x [H, R, P] -> [.., H, R, P] in the io dtype (fp32 product, rounded)."""
    return (v.float().unsqueeze(-2) * w).to(io)


def _workload(b, H, G, P, N, R, T, io, seed):
    inp = inputs.make_scan_inputs(b, T, H, G, P, N, R, io_dtype=io, theta_max=math.pi / 8,
                                  seed=seed, h0_random=True, carry_prev=True)
    x1 = inp["x"][:, :, :, 0, :].contiguous()
    z1 = inputs.make_gate((b, T, H, P), io_dtype=io, seed=seed)
    wx, wz = inputs.make_expand(H, R, P, seed=seed)
    return inp, x1, z1, wx, wz


def _run(inp, d, T, Q, x, ex, flags=0, calls=1):
    g = {k: v.cuda() for k, v in inp.items()}
    st = m3.State(d)
    st.h.copy_(g["h0"])
    st.x_prev.copy_(g["x_prev"])
    st.B_prev.copy_(g["B_prev"])
    b, H, R, P = d.batch, d.nheads, d.rank, d.headdim
    y = torch.full((b, T, H, R, P), float("nan"), dtype=g["x"].dtype, device="cuda")
    bounds = np.linspace(0, T, calls + 1).astype(int)
    ws = m3.alloc_workspace_ex(d, int(np.diff(bounds).max()), Q, ex)
    for c in range(calls):
        lo, hi = int(bounds[c]), int(bounds[c + 1])
        sl = {k: g[k][:, lo:hi].contiguous() for k in KEYS if k != "x"}
        xc = x[:, lo:hi].contiguous()
        exc = ex
        if ex is not None and ex.z is not None:
            exc = m3.Extras(z=ex.z[:, lo:hi].contiguous(), x_expand=ex.x_expand,
                            z_expand=ex.z_expand)
        yc = torch.empty((b, hi - lo, H, R, P), dtype=g["x"].dtype, device="cuda")
        m3.m3_scan_fwd_ex(d, hi - lo, Q, xc, sl["B"], sl["C"], sl["dt"], sl["A"], sl["lam"],
                          sl["theta"], g["D"], exc, st, yc, ws, flags)
        assert m3.m3_query_status(ws) == m3.M3_OK
        y[:, lo:hi] = yc
    torch.cuda.synchronize()
    return y, st


CASES = [
    # (b, H, G, P, N, R, T, chunk, io, tol, flags, x_exp, z_mode) z_mode: None | "plain" | "exp"
    (1, 4, 1, 64, 64, 4, 150, 64, torch.bfloat16, 2e-2, 0, True, None),     # R=4, 32-token tiles
    (1, 4, 1, 64, 64, 4, 150, 64, torch.bfloat16, 2e-2, 0, True, "exp"),
    (1, 4, 1, 64, 64, 4, 96, 16, torch.bfloat16, 2e-2, 0, True, "plain"),   # 16-token tiles
    (1, 4, 1, 64, 64, 4, 100, 32, torch.bfloat16, 2e-2, 0, False, "exp"),   # gate only
    (2, 4, 2, 64, 64, 2, 90, 32, torch.bfloat16, 2e-2, 0, True, "exp"),     # R=2, G=2
    (1, 4, 1, 64, 128, 1, 300, 64, torch.bfloat16, 2e-2, 0, True, "exp"),   # R=1, ragged
    (1, 4, 1, 64, 64, 4, 70, 32, torch.bfloat16, 2e-2, m3.M3_FLAG_FORCE_SIMT, True, "exp"),
    (1, 3, 3, 8, 6, 3, 40, 16, torch.float32, 1e-5, 0, True, "exp"),        # fp32 sequential
]


def _id(c):
    return (f"N{c[4]}R{c[5]}T{c[6]}Q{c[7]}{'f32' if c[8] == torch.float32 else 'bf16'}"
            f"{'S' if c[10] else ''}{'x' if c[11] else ''}{c[12] or ''}")


@pytest.mark.parametrize("case", CASES, ids=[_id(c) for c in CASES])
def test_expanded_scan_matches_oracle(case):
    b, H, G, P, N, R, T, Q, io, tol, flags, xe, zm = case
    inp, x1, z1, wx, wz = _workload(b, H, G, P, N, R, T, io, seed=31)
    d = m3.Dims(b, H, G, P, N, R, m3.io_dtype_of(io))
    zfull = inputs.make_gate((b, T, H, R, P), io_dtype=io, seed=31)
    z = None if zm is None else (z1 if zm == "exp" else zfull)
    ex = m3.Extras(z=None if z is None else z.cuda(), x_expand=wx.cuda() if xe else None,
                   z_expand=wz.cuda() if zm == "exp" else None)
    x = (x1 if xe else inp["x"]).cuda()
    y, st = _run(inp, d, T, Q, x, ex, flags)
    ko = dict(D=f64(inp["D"]), h0=f64(inp["h0"]), x_prev=f64(inp["x_prev"]),
              B_prev=f64(inp["B_prev"]), z=None if z is None else f64(z),
              x_expand=f64(wx) if xe else None, z_expand=f64(wz) if zm == "exp" else None)
    yo, ho, xpo, _ = oracle.scan(f64(x1 if xe else inp["x"]),
                                 *(f64(inp[k]) for k in KEYS[1:]), **ko)
    yg = f64(y)
    assert np.all(np.isfinite(yg))
    assert rel_slices(yg, yo, (1, 3, 4)) <= tol
    assert rel_slices(f64(st.h), ho, (2, 3)) <= tol
    # the carried x is the expanded last token, in the io dtype
    xtol = 2.0 ** -8 if io == torch.bfloat16 else 1e-6
    assert rel_slices(f64(st.x_prev), xpo, (2, 3)) <= xtol

    # on chip expansion == the plain call on the expanded io-dtype tensors, bit for bit
    xfull = _host_expand(x1, wx, io) if xe else inp["x"]
    zref = None if z is None else (_host_expand(z1, wz, io) if zm == "exp" else zfull)
    y2, st2 = _run(inp, d, T, Q, xfull.cuda(),
                   None if zref is None else m3.Extras(z=zref.cuda()), flags)
    assert torch.equal(y, y2)
    assert torch.equal(st.h, st2.h) and torch.equal(st.x_prev, st2.x_prev)


def test_expanded_scan_chained_calls():
    """Three chained expanded calls equal one oracle call: the state carries X_{T-1}."""
    b, H, G, P, N, R, T, Q = 1, 4, 1, 64, 64, 4, 200, 64
    inp, x1, z1, wx, wz = _workload(b, H, G, P, N, R, T, torch.bfloat16, seed=37)
    d = m3.Dims(b, H, G, P, N, R, m3.M3_BF16)
    ex = m3.Extras(z=z1.cuda(), x_expand=wx.cuda(), z_expand=wz.cuda())
    y, st = _run(inp, d, T, Q, x1.cuda(), ex, calls=3)
    yo, ho, _, _ = oracle.scan(f64(x1), *(f64(inp[k]) for k in KEYS[1:]), D=f64(inp["D"]),
                               h0=f64(inp["h0"]), x_prev=f64(inp["x_prev"]),
                               B_prev=f64(inp["B_prev"]), z=f64(z1), x_expand=f64(wx),
                               z_expand=f64(wz))
    assert rel_slices(f64(y), yo, (1, 3, 4)) <= 2e-2
    assert rel_slices(f64(st.h), ho, (2, 3)) <= 2e-2


@pytest.mark.parametrize("shape,io,tol", [
    ((4, 8, 1, 64, 128, 1), torch.bfloat16, 2e-2),
    ((4, 8, 2, 64, 64, 4), torch.bfloat16, 2e-2),
    ((2, 6, 3, 8, 6, 3), torch.float32, 1e-5),
    ((3, 4, 2, 64, 64, 2), torch.float32, 1e-5),
])
def test_expanded_decode_matches_oracle(shape, io, tol):
    b, H, G, P, N, R = shape
    steps = 5
    inp = inputs.make_decode_inputs(b, H, G, P, N, R, tokens=steps, io_dtype=io, seed=41)
    x1 = inp["x"][:, :, :, 0, :].contiguous()
    z1 = inputs.make_gate((steps, b, H, P), io_dtype=io, seed=41)
    wx, wz = inputs.make_expand(H, R, P, seed=41)
    d = m3.Dims(b, H, G, P, N, R, m3.io_dtype_of(io))
    st = m3.State(d)
    st.h.copy_(inp["h0"])
    st.x_prev.copy_(inp["x_prev"])
    st.B_prev.copy_(inp["B_prev"])
    g = {k: inp[k].cuda() for k in KEYS}
    xg, zg, D = x1.cuda(), z1.cuda(), inp["D"].cuda()
    ex = m3.Extras(x_expand=wx.cuda(), z_expand=wz.cuda())
    h, xp, bp = f64(inp["h0"]), f64(inp["x_prev"]), f64(inp["B_prev"])
    for t in range(steps):
        y = torch.empty((b, H, R, P), dtype=io, device="cuda")
        ex.z = zg[t]
        m3.m3_decode_step_ex(d, xg[t], *(g[k][t] for k in KEYS[1:]), D, ex, st, y)
        yo, h, xp, bp = oracle.decode_step(f64(x1[t]), *(f64(inp[k][t]) for k in KEYS[1:]),
                                           f64(inp["D"]), h, xp, bp, z=f64(z1[t]),
                                           x_expand=f64(wx), z_expand=f64(wz))
        assert rel_slices(f64(y), yo, (2, 3)) <= tol
    assert rel_slices(f64(st.h), h, (2, 3)) <= tol
    # x_prev holds the expanded last token exactly as the io dtype rounds it
    assert torch.equal(st.x_prev.cpu(), _host_expand(x1[-1], wx, io))
